// Forward DCNv2 on sm_100a tensor cores, bfloat16 in / float32 accumulate.
//
// The layer is the dense contraction Y[P x Cout] = Col[P x K*K*Cin] * W^T with
// P = B*Ho*Wo output pixels, where a row of Col holds the modulated bilinear
// samples m * x(p0 + p_k + dp_k) of one output pixel (the im2col view of the
// deformable convolution: the "Deformable ConvNets" notes, im2col appendix and
// the y(p0) equations). Col is never written to HBM:
//
//   * producer warps (8) gather every chunk (one tap, 64 channels): each lane
//     loads the four channel-contiguous NHWC neighbours of a sample as 32-byte
//     vectors (16 channels), blends them with the bilinear weights times the
//     mask, and stores the bf16 result straight into a shared-memory A tile laid
//     out in the UMMA 128-byte-swizzle K-major canonical form; a thread owns two
//     rows and issues the next chunk's loads for a row right after blending it;
//   * one TMA warp stages the matching weight tile [N x 64] of W = [Cout, K*K*Cin];
//   * one MMA warp issues tcgen05.mma (M=128, N<=256, K=16) into TMEM;
//   * four epilogue warps build the sampling records (bilinear weights times the
//     mask, top-left neighbour, neighbours to read) one (tile, group) epoch ahead
//     of the producers, and read the accumulator back with tcgen05.ld, add the
//     bias and store bf16 NHWC rows.
//
// The K loop runs over (group, 64-channel chunk, tap), taps innermost, so that
// consecutive chunks gather from the same 128-byte channel slice of nearby
// pixels while it is in L1. Work is split stream-K style: the (tile, chunk)
// units are divided evenly over one persistent CTA per SM (no CTA starting in
// the last units of a tile); a tile that two or more CTAs share is summed from
// float32 partial tiles in the workspace, in contributor order, by the CTA that
// finishes it last (counted with an atomic per tile; no CTA waits on another).
// Every wait is bounded and reports a timeout through the status word.
#include <cudaTypedefs.h>
#include "fwd_common.cuh"

namespace dcn {
namespace {

constexpr int A_STAGE_BYTES = BM * BK * 2;
constexpr int NUM_PROD_WARPS = 8;
constexpr int TMA_WARP = 4, MMA_WARP = 5, PROD_WARP0 = 6;  // warps 0-3: epilogue
constexpr int NUM_THREADS = (PROD_WARP0 + NUM_PROD_WARPS) * 32;
constexpr int NUM_PROD_THREADS = NUM_PROD_WARPS * 32;
constexpr int SLICE = 16;                                   // channels one lane gathers per sample (32 bytes)
constexpr int LANES_PER_ROW = BK / SLICE;
constexpr int ROW_STEP = NUM_PROD_THREADS / LANES_PER_ROW;  // rows between a thread's two rows
static_assert(ROW_STEP % 8 == 0, "a thread's rows must share their swizzle phase");
static_assert(2 * ROW_STEP == BM, "two rows per producer thread and chunk");
#ifndef DCN_FWD_MAX_STAGES
#define DCN_FWD_MAX_STAGES 3
#endif

// WIDE: x is 32-byte aligned and Cin, Cg are multiples of 16, so a lane's
// 16-channel slice is one 32-byte load.
template <bool WIDE>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    dcn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmap_w, const FwdArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Shape& s = a.s;

    uint8_t* sA = smem;
    uint8_t* sB = smem + a.b_off;
    TapRec* s_rec = reinterpret_cast<TapRec*>(smem + a.info_off);  // two buffers of BM * K2 records
    int2* s_tap = reinterpret_cast<int2*>(smem + a.row_off);        // per tap: (i*dil, j*dil)
    long long* s_starts = reinterpret_cast<long long*>(s_tap + 32);   // [ctas + 1] first unit of each CTA
    float* s_bias = reinterpret_cast<float*>(s_starts + MAX_CTAS + 2);  // [2][512] bias of a tile's columns
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + a.bar_off);
    // barrier slots
    uint64_t* full_a = bars;
    uint64_t* tail_bar = bars + MAX_STAGES;  // bulk copy of other CTAs' partials for the last segment
    uint64_t* empty = bars + 2 * MAX_STAGES;
    uint64_t* acc_full = bars + 3 * MAX_STAGES;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* drain = acc_empty + 2;
    uint64_t* rec_full = drain + 1;    // [2] records of an epoch built
    uint64_t* rec_empty = rec_full + 2;  // [2] every producer warp done with an epoch's records
    uint64_t* rec0_bar = rec_empty + 2;  // the first epoch's records, built by all warps
    uint64_t* epi_bar = rec0_bar + 1;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(epi_bar + 1);
    volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
    volatile int* s_last = s_abort + 1;  // [2], by segment parity

    if (threadIdx.x == 0) {
        for (int i = 0; i < a.stages; ++i) {
            // a stage is full when every producer warp and the weight TMA have arrived
            ptx::mbar_init(ptx::smem_u32(&full_a[i]), NUM_PROD_WARPS + 1);
            ptx::mbar_init(ptx::smem_u32(&empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(ptx::smem_u32(&acc_full[i]), 1);
            ptx::mbar_init(ptx::smem_u32(&acc_empty[i]), 4);
        }
        ptx::mbar_init(ptx::smem_u32(drain), 1);
        ptx::mbar_init(ptx::smem_u32(tail_bar), 1);
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(ptx::smem_u32(&rec_full[i]), 4);
            ptx::mbar_init(ptx::smem_u32(&rec_empty[i]), NUM_PROD_WARPS);
        }
        ptx::mbar_init(ptx::smem_u32(rec0_bar), NUM_PROD_WARPS + 4);
        ptx::mbar_init(ptx::smem_u32(epi_bar), 4);
        *s_abort = 0;
        s_last[0] = s_last[1] = 0;
        ptx::fence_mbar_init();
    }
    if (threadIdx.x < s.K2) {
        const int i = threadIdx.x / s.K;
        s_tap[threadIdx.x] = make_int2(i * s.dil, (threadIdx.x - i * s.K) * s.dil);
    }
    for (int c = threadIdx.x; c <= a.ctas; c += NUM_THREADS) s_starts[c] = unit_begin(c, a);
    if (warp == MMA_WARP) {
        ptx::tmem_alloc(ptx::smem_u32(s_tmem), (uint32_t)a.tmem_cols);
        ptx::tmem_relinquish();
    }
    if (warp == TMA_WARP && lane == 0) ptx::prefetch_tmap(&tmap_w);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *s_tmem;

    const int cta = blockIdx.x;
    const long long ubeg = s_starts[cta], uend = s_starts[cta + 1];
    const SegList L = seg_list(ubeg, uend, a.U);
    if (warp >= PROD_WARP0) {
        // ------------------------------------------------------ producers --
        // All producer warps work on every chunk: 4 lanes cover the 128-byte
        // channel slice of one row (16 channels each), and a thread owns rows r0
        // and r0 + ROW_STEP, which share one swizzle phase. The loads of the next
        // chunk's row are issued right after this chunk's row is blended, so they
        // are in flight while the other row is blended and stored.
        const int ptid = threadIdx.x - PROD_WARP0 * 32;
        const int j4 = ptid % LANES_PER_ROW, r0 = ptid / LANES_PER_ROW;
        const int r1 = r0 + ROW_STEP;
        const uint32_t swz0 = (uint32_t)(((2 * j4) ^ (r0 & 7)) << 4);      // 16-byte chunk 2*j4 of the row
        const uint32_t swz1 = (uint32_t)(((2 * j4 + 1) ^ (r0 & 7)) << 4);  // chunk 2*j4 + 1
        const long long cin2 = (long long)s.Cin * 2, rp2 = (long long)s.W * cin2;
        const uint8_t* zb = reinterpret_cast<const uint8_t*>(g_zero_slice);
#ifdef DCN_CHECKED
        const size_t xbytes = (size_t)s.B * s.H * s.W * s.Cin * sizeof(bf16);  // range-checked build
#endif
        bool ok = true;
        // the first epoch's records are built by all warps together
        if (L.ns > 0) {
            const Seg s0 = seg_at(L, 0);
            build_records(a, s0.t / a.n_tiles, s0.k0 / (a.nq * s.K2), ptid & (BM - 1), 1 + (ptid >> 7), s_rec, s_tap);
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(rec0_bar));
            ok = ptx::mbar_wait(ptx::smem_u32(rec0_bar), 0, s_abort, a.status, WAIT_LIMIT);
        }
        // issue cursor: the chunk whose loads are issued next
        int isi = 0, ik = 0, ik1 = 0, icur_g = -1, iepoch = 0;
        Chunk ich{0, 0, 0};
        // shared-memory address of the current epoch's records: read with ld.shared,
        // which does not queue behind the gathers in the global-load path
        uint32_t irecs = ptx::smem_u32(s_rec);
        if (L.ns > 0) {
            const Seg s0 = seg_at(L, 0);
            ik = s0.k0;
            ik1 = s0.k1;
            ich = chunk_of(ik, a);
            icur_g = ich.g;
        }
        // loads of row `row` of the cursor chunk into v, its weights into w
        auto issue = [&](uint32_t(&v)[4][8], uint32_t(&w)[2], int row) {
            const int cg = ich.q * BK + j4 * SLICE;  // first channel of this lane's slice, within the group
            const uint32_t cmask = cg < s.Cg ? 0xFu : 0u;
            const bool hi_ok = cg + 8 < s.Cg;      // upper 8 channels present (narrow loads only)
            const uint8_t* xc = reinterpret_cast<const uint8_t*>(a.x + ich.g * s.Cg + cg);
            const uint4 rc = ptx::lds_v4(irecs + (uint32_t)((row * s.K2 + ich.tap) * (int)sizeof(TapRec)));
            w[0] = rc.x;  // TapRec::w01_00
            w[1] = rc.y;  // TapRec::w11_10
            const uint32_t vm = rc.w & cmask;  // TapRec::vmask
            const uint8_t* p = xc + (long long)(int)rc.z * cin2;  // TapRec::base
            const uint8_t* pc[4] = {p, p + cin2, p + rp2, p + rp2 + cin2};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
#ifdef DCN_CHECKED
                const bool rd = ((vm >> c) & 1u) &&
                                ptx::in_range(pc[c], (WIDE || hi_ok) ? 32 : 16, a.x, xbytes, a.status);
#else
                const bool rd = (vm >> c) & 1u;
#endif
                load_slice<WIDE>(v[c], rd ? pc[c] : zb, (rd && hi_ok) ? pc[c] + 16 : zb);
            }
        };
        // moves the cursor to the next chunk; at a new epoch (tile or group) releases the
        // previous records and waits for the new ones
        auto advance = [&]() -> bool {
            ++ik;
            if (++ich.tap == s.K2) {
                ich.tap = 0;
                if (++ich.q == a.nq) {
                    ich.q = 0;
                    ++ich.g;
                }
            }
            if (ik == ik1) {
                const Seg sn = seg_at(L, ++isi);
                ik = sn.k0;
                ik1 = sn.k1;
                ich = chunk_of(ik, a);
                icur_g = -1;
            }
            if (ich.g != icur_g) {
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&rec_empty[iepoch & 1]));
                ++iepoch;
                const int b = iepoch & 1;
                const uint32_t par = (uint32_t)(b ? (iepoch >> 1) : ((iepoch >> 1) - 1)) & 1u;
                if (!ptx::mbar_wait(ptx::smem_u32(&rec_full[b]), par, s_abort, a.status, WAIT_LIMIT)) return false;
                irecs = ptx::smem_u32(s_rec + b * BM * s.K2);
                icur_g = ich.g;
            }
            return true;
        };
        const long long total = uend - ubeg;  // chunks of this CTA
        uint32_t va[4][8], vb[4][8], wa[2], wb[2];
        if (ok && total > 0) {
            issue(va, wa, r0);
            issue(vb, wb, r1);
        }
        int stage = 0;
        uint32_t phase = 0;
        for (long long n = 0; n < total && ok; ++n) {
            if (!ptx::mbar_wait(ptx::smem_u32(&empty[stage]), phase ^ 1, s_abort, a.status, WAIT_LIMIT)) {
                ok = false;
                break;
            }
            const uint32_t a_stage = ptx::smem_u32(sA + stage * A_STAGE_BYTES);
            const bool more = n + 1 < total;
            {
                uint32_t r[8];
                blend16(r, va, wa[0], wa[1]);
                ptx::sts_v4(a_stage + r0 * 128 + swz0, make_uint4(r[0], r[1], r[2], r[3]));
                ptx::sts_v4(a_stage + r0 * 128 + swz1, make_uint4(r[4], r[5], r[6], r[7]));
            }
            if (more) {
                if (!advance()) {
                    ok = false;
                    break;
                }
                issue(va, wa, r0);
            }
            {
                uint32_t r[8];
                blend16(r, vb, wb[0], wb[1]);
                ptx::sts_v4(a_stage + r1 * 128 + swz0, make_uint4(r[0], r[1], r[2], r[3]));
                ptx::sts_v4(a_stage + r1 * 128 + swz1, make_uint4(r[4], r[5], r[6], r[7]));
            }
            if (more) issue(vb, wb, r1);
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&full_a[stage]));
            if (++stage == a.stages) {
                stage = 0;
                phase ^= 1;
            }
        }
    } else if (warp == TMA_WARP) {
        // ------------------------------------------------------- weights --
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued = 0, issued_par = 0;  // per stage: a load was issued / parity of the last one
            const uint32_t bytes = (uint32_t)(a.nsub * a.box_rows * BK * 2);
            bool ok = true;
            for (int si = 0; si < L.ns && ok; ++si) {
                const Seg sg = seg_at(L, si);
                const int n0 = (sg.t % a.n_tiles) * a.bn_total;
                for (int k = sg.k0; k < sg.k1; ++k) {
                    const Chunk ch = chunk_of(k, a);
                    if (!ptx::mbar_wait(ptx::smem_u32(&empty[stage]), phase ^ 1, s_abort, a.status, WAIT_LIMIT)) {
                        ok = false;
                        break;
                    }
                    const int xk = ch.tap * s.Cin + ch.g * s.Cg + ch.q * BK;
                    const uint32_t fb = ptx::smem_u32(&full_a[stage]);
                    ptx::mbar_arrive_expect_tx(fb, bytes);
                    for (int sub = 0; sub < a.nsub; ++sub)
                        ptx::tma_load_2d(ptx::smem_u32(sB + stage * a.b_stage_bytes + sub * a.box_rows * 128),
                                         &tmap_w, fb, xk, n0 + sub * 256);
                    issued |= 1u << stage;
                    issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == a.stages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            if (*s_abort) {
                // wait (bounded) for loads still in flight before shared memory is released
                volatile int dummy = 0;
                for (int i = 0; i < a.stages; ++i)
                    if ((issued >> i) & 1u)
                        ptx::mbar_wait(ptx::smem_u32(&full_a[i]), (issued_par >> i) & 1u, &dummy, nullptr,
                                       WAIT_LIMIT);
            }
        }
        __syncwarp();
    } else if (warp == MMA_WARP) {
        // ----------------------------------------------------------- MMA --
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            const uint32_t idesc0 = ptx::idesc_bf16_f32(BM, a.nsub == 1 ? a.bn_total : 256);
            const uint32_t idesc1 = ptx::idesc_bf16_f32(BM, a.nsub == 1 ? 16 : a.bn_total - 256);
            const uint32_t a0 = ptx::smem_u32(sA), b0 = ptx::smem_u32(sB);
            bool ok = true;
            for (int seg = 0; seg < L.ns && ok; ++seg) {
                const Seg sg = seg_at(L, seg);
                const int abuf = a.acc_cols ? (seg & 1) : 0;
                const uint32_t aphase = a.acc_cols ? ((seg >> 1) & 1) : (seg & 1);
                if (!ptx::mbar_wait(ptx::smem_u32(&acc_empty[abuf]), aphase ^ 1, s_abort, a.status, WAIT_LIMIT)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t d = tmem_base + (uint32_t)(abuf * a.acc_cols);
                for (int k = sg.k0; k < sg.k1; ++k) {
                    if (!ptx::mbar_wait(ptx::smem_u32(&full_a[stage]), phase, s_abort, a.status, WAIT_LIMIT)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t as = a0 + stage * A_STAGE_BYTES, bs = b0 + stage * a.b_stage_bytes;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint32_t acc = (k > sg.k0 || kk > 0) ? 1u : 0u;
                        ptx::mma_bf16(d, ptx::sw128_desc(as + kk * 32), ptx::sw128_desc(bs + kk * 32), idesc0, acc);
                        if (a.nsub == 2)
                            ptx::mma_bf16(d + 256, ptx::sw128_desc(as + kk * 32),
                                          ptx::sw128_desc(bs + a.box_rows * 128 + kk * 32), idesc1, acc);
                    }
                    ptx::mma_commit(ptx::smem_u32(&empty[stage]));
                    if (++stage == a.stages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                ptx::mma_commit(ptx::smem_u32(&acc_full[abuf]));
            }
            // all MMAs issued by this thread complete before TMEM is released
            ptx::mma_commit(ptx::smem_u32(drain));
            volatile int dummy = 0;
            ptx::mbar_wait(ptx::smem_u32(drain), 0, &dummy, a.status, WAIT_LIMIT);
        }
        __syncwarp();
    } else {
        // ------------------------------------------- records and epilogue --
        // These four warps also build the sampling records, one epoch (a run of
        // the CTA's chunks with one tile and group) ahead of the producers, in
        // two buffers. Before the epilogue of a segment they build every epoch
        // of that segment and the first one of the next; building epoch e waits
        // only for the producers to release epoch e - 2, which needs no
        // epilogue of this segment, so the order cannot deadlock.
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const int per_g = a.nq * s.K2;
        uint32_t ephase = 0;
        int rec_epoch = 0;
        int rseg = 0, rk = L.ns > 0 ? seg_at(L, 0).k0 : 0;  // next epoch to build: its segment and first unit
        bool ok = true;
        for (int seg = 0; seg < L.ns && ok; ++seg) {
            const Seg sg = seg_at(L, seg);
            const int t = sg.t;
            while (rseg < L.ns && (rseg <= seg || (rseg == seg + 1 && rk == seg_at(L, rseg).k0))) {
                const Seg rs = seg_at(L, rseg);
                const int b = rec_epoch & 1;
                if (rec_epoch >= 2 && !ptx::mbar_wait(ptx::smem_u32(&rec_empty[b]), ((rec_epoch - 2) >> 1) & 1, s_abort,
                                                      a.status, WAIT_LIMIT)) {
                    ok = false;
                    break;
                }
                const int rg = rk / per_g;
                // the first epoch is shared with the producer warps
                build_records(a, rs.t / a.n_tiles, rg, row, rec_epoch == 0 ? 0 : -1, s_rec + b * BM * s.K2, s_tap);
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(rec_epoch == 0 ? rec0_bar : &rec_full[b]));
                rk = min((rg + 1) * per_g, rs.k1);
                if (rk >= rs.k1 && ++rseg < L.ns) rk = seg_at(L, rseg).k0;
                ++rec_epoch;
            }
            if (!ok) break;

            const int abuf = a.acc_cols ? (seg & 1) : 0;
            const uint32_t aphase = a.acc_cols ? ((seg >> 1) & 1) : (seg & 1);
            const bool full = (sg.k0 == 0 && sg.k1 == a.U);
            const bool last_proc = seg == L.ns - 1;  // the pipeline is idle after this segment's accumulator
            const long long tu0 = (long long)t * a.U;
            int c_lo = cta, c_hi = cta;
            if (!full) {
                c_lo = cta_of_unit(tu0, s_starts, a.ctas);
                c_hi = cta_of_unit(tu0 + a.U - 1, s_starts, a.ctas);
            }
            // Thread 0 learns whether every other contributor of this tile has
            // published its partial: one read before the accumulator is ready
            // and, for the CTA's last segment, a fresh one after.
            int cnt = -1;
            if (!full && threadIdx.x == 0) cnt = ptx::ld_relaxed_gpu(a.counters + t);
            if (!ptx::mbar_wait(ptx::smem_u32(&acc_full[abuf]), aphase, s_abort, a.status, WAIT_LIMIT)) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            const int mt = t / a.n_tiles, n0 = (t % a.n_tiles) * a.bn_total;
            const int ncols = min(a.bn_total, s.Cout - n0);
            if (threadIdx.x == 0) {
                int last = full ? 1 : 0;
                if (!full) {
                    if (cnt != c_hi - c_lo && last_proc) cnt = ptx::ld_relaxed_gpu(a.counters + t);
                    last = cnt == c_hi - c_lo;
                    if (last) ptx::fence_acq_rel_gpu();  // the partials read below follow the counter
                }
                s_last[seg & 1] = last;
            }
            float* sbias = s_bias + (seg & 1) * 512;  // by segment parity, like s_last
            if (a.bias)
                for (int i = threadIdx.x; i < ncols; i += 4 * 32) sbias[i] = __bfloat162float(a.bias[n0 + i]);
            if (!epi_sync(epi_bar, ephase, s_abort, a.status)) {
                ok = false;
                break;
            }
            const float* sb = a.bias ? sbias : nullptr;
            const int p = strip_to_raster(mt * BM + row, a);
            const uint32_t taddr = tmem_base + (uint32_t)(abuf * a.acc_cols) + ((uint32_t)(quarter * 32) << 16);
            bf16* ycol0 = a.y + n0;  // y[pixel, n0 + col] = ycol0[pixel * Cout + col]
            if (s_last[seg & 1]) {
                // y = this CTA's accumulator + the other contributors' partials + bias. In
                // the CTA's last segment the pipeline buffers are idle, so when the
                // partials fit there they are bulk-copied in and read from shared memory.
                const uint32_t tile_bytes = (uint32_t)BM * a.bn_total * 4;
                const bool staged = !full && last_proc &&
                                    (uint32_t)(c_hi - c_lo) * tile_bytes <= a.b_off + a.stages * a.b_stage_bytes;
                if (staged) {
                    if (threadIdx.x == 0) {
                        ptx::fence_proxy_async_all();
                        const uint32_t tb = ptx::smem_u32(tail_bar);
                        ptx::mbar_arrive_expect_tx(tb, (uint32_t)(c_hi - c_lo) * tile_bytes);
                        uint32_t dst = ptx::smem_u32(smem);
                        for (int c = c_lo; c <= c_hi; ++c) {
                            if (c == cta) continue;
                            const uint8_t* src = reinterpret_cast<const uint8_t*>(partial_base(a, s_starts, c, tu0, 0));
                            for (uint32_t o = 0; o < tile_bytes; o += 16384u)
                                ptx::bulk_load(dst + o, src + o, min(16384u, tile_bytes - o), tb);
                            dst += tile_bytes;
                        }
                    }
                    if (!ptx::mbar_wait(ptx::smem_u32(tail_bar), 0, s_abort, a.status, WAIT_LIMIT)) {
                        ok = false;
                        break;
                    }
                }
                // In the CTA's last segment the output rows are staged for full-line stores
                // in the idle pipeline buffers, after any staged partials (4 warps x 4 KB).
                const uint32_t yoff = staged ? (uint32_t)(c_hi - c_lo) * tile_bytes : 0u;
                const uint32_t ybuf = (last_proc && yoff + 4 * 4096 <= a.b_off + a.stages * a.b_stage_bytes)
                                          ? ptx::smem_u32(smem + yoff) + quarter * 4096
                                          : 0u;
                combine_rows(taddr, ncols, c_lo, c_hi, cta, staged, [&](int c) -> const float* {
                    // staged partials are packed in contributor order without this CTA's
                    if (staged) return reinterpret_cast<const float*>(smem + (size_t)(c - c_lo - (c > cta)) * tile_bytes) + row * 4;
                    return partial_base(a, s_starts, c, tu0, row);
                }, sb, ybuf, ycol0, p, s.Cout);
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&acc_empty[abuf]));
                if (!full && threadIdx.x == 0) a.counters[t] = 0;
            } else {
                // publish this CTA's partial tile, then count it in; the accumulator
                // stays in TMEM until it is known whether this CTA finishes the tile
                float* dst = const_cast<float*>(partial_base(a, s_starts, cta, tu0, row));
                tmem_rows<true>(taddr, a.bn_total, [&](uint32_t(&r)[32], int cc) {
                    float* b = dst + (size_t)(cc >> 5) * 8 * BM * 4;
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        *reinterpret_cast<uint4*>(b + q * BM * 4) = make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
                });
                __threadfence();
                if (!epi_sync(epi_bar, ephase, s_abort, a.status)) {
                    ok = false;
                    break;
                }
                if (threadIdx.x == 0) s_last[seg & 1] = (atomicAdd(a.counters + t, 1) == c_hi - c_lo) ? 1 : 0;
                if (!epi_sync(epi_bar, ephase, s_abort, a.status)) {
                    ok = false;
                    break;
                }
                if (s_last[seg & 1]) {
                    // every other contributor's partial is in the workspace
                    __threadfence();
                    combine_rows(taddr, ncols, c_lo, c_hi, cta, false, [&](int c) -> const float* {
                        return partial_base(a, s_starts, c, tu0, row);
                    }, sb, 0u, ycol0, p, s.Cout);
                    if (threadIdx.x == 0) a.counters[t] = 0;
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&acc_empty[abuf]));
            }
        }
    }

    // ------------------------------------------------------------ teardown --
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, (uint32_t)a.tmem_cols);
    }
}

// ------------------------------------------------------------------- host --

struct Plan {
    bool ok;
    int bn_total, n_tiles, m_tiles, tiles, nq, U, ctas, nsub, box_rows, stages, acc_cols, tmem_cols;
    int sw, nf, wl, snap;
    long long total_units;
    uint32_t b_off, info_off, row_off, bar_off, b_stage_bytes, smem_bytes;
    size_t ws_partials, ws_counters_off, ws_bytes;
};

Plan make_plan(const Shape& s, int sms) {
    Plan pl{};
    pl.ok = false;
    if (s.Cin % 8 || s.Cg % 8 || s.Cout % 8 || s.K2 > 25) return pl;
    pl.bn_total = std::min(512, (s.Cout + 31) / 32 * 32);
    const StreamK k = plan_stream_k(s, pl.bn_total, sms);
    pl.n_tiles = k.n_tiles;
    pl.m_tiles = k.m_tiles;
    pl.tiles = k.tiles;
    pl.nq = k.nq;
    pl.sw = k.sw;
    pl.nf = k.nf;
    pl.wl = k.wl;
    pl.U = k.U;
    pl.total_units = k.total_units;
    pl.ctas = k.ctas;
    pl.snap = k.snap;
    pl.nsub = pl.bn_total > 256 ? 2 : 1;
    pl.box_rows = pl.nsub == 1 ? pl.bn_total : 256;
    pl.b_stage_bytes = (uint32_t)(pl.nsub * pl.box_rows * 128);
    if (pl.nsub == 1) {
        int cols = 32;
        while (cols < 2 * pl.bn_total) cols *= 2;
        pl.tmem_cols = cols;
        pl.acc_cols = cols / 2;
    } else {
        pl.tmem_cols = 512;
        pl.acc_cols = 0;
    }
    const uint32_t info_bytes = (uint32_t)(2 * BM * s.K2 * sizeof(TapRec));  // two record buffers
    const uint32_t fixed = info_bytes + 256 + (MAX_CTAS + 2) * 8 + 4096 + (3 * MAX_STAGES + 14) * 8 + 16 + 1024;
    const uint32_t budget = 227 * 1024;
    const uint32_t stage_bytes = A_STAGE_BYTES + pl.b_stage_bytes;
    int st = (int)((budget - fixed) / stage_bytes);
    st = std::min(st, DCN_FWD_MAX_STAGES);
    if (st < 2) return pl;
    pl.stages = st;
    pl.b_off = (uint32_t)(st * A_STAGE_BYTES);
    pl.info_off = pl.b_off + (uint32_t)st * pl.b_stage_bytes;
    pl.row_off = pl.info_off + info_bytes;
    // taps, CTA start table, bias of one tile
    pl.bar_off = pl.row_off + (uint32_t)(32 * sizeof(int2) + (MAX_CTAS + 2) * sizeof(long long) + 2 * 512 * sizeof(float));
    pl.smem_bytes = pl.bar_off + (3 * MAX_STAGES + 14) * 8 + 16 + 1024;
    if (pl.smem_bytes > budget) return pl;
    pl.ws_partials = (size_t)pl.ctas * 2 * BM * pl.bn_total * sizeof(float);
    pl.ws_counters_off = (pl.ws_partials + 255) & ~(size_t)255;
    pl.ws_bytes = pl.ws_counters_off + (size_t)pl.tiles * sizeof(int);
    pl.ok = true;
    return pl;
}

}  // namespace

// Layers with Cout <= 256 run the kernel of fwd_tc_ts.cu (gathered operand in
// tensor memory); wider ones run this file's kernel.
bool fwd_tc_supported(const Shape& s) { return fwd_ts_supported(s) || make_plan(s, num_sms()).ok; }

const char* fwd_tc_variant(const Shape& s) {
    return fwd_ts_supported(s) ? "tcgen05_gather_tmem" : "tcgen05_gather";
}

size_t fwd_tc_workspace(const Shape& s) {
    if (fwd_ts_supported(s)) return fwd_ts_workspace(s);
    Plan pl = make_plan(s, num_sms());
    return pl.ok ? pl.ws_bytes : 0;
}

cudaError_t fwd_tc(const Shape& s, const void* x, const void* off, const void* mask, const void* w, const void* bias,
                   void* y, void* ws, size_t ws_bytes, unsigned* status, cudaStream_t st, int* launches) {
    if (fwd_ts_supported(s)) {
        const cudaError_t e = fwd_ts(s, x, off, mask, w, bias, y, ws, ws_bytes, status, st, launches);
        if (e != cudaErrorNotSupported) return e;
        (void)cudaGetLastError();  // the build's register layout does not fit that kernel: run this one
    }
    Plan pl = make_plan(s, num_sms());
    if (!pl.ok || ws_bytes < pl.ws_bytes || !ws) return cudaErrorInvalidValue;
    auto encode = get_encode();
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap map;
    cuuint64_t dims[2] = {(cuuint64_t)s.KC, (cuuint64_t)s.Cout};
    cuuint64_t strides[1] = {(cuuint64_t)s.KC * 2};
    cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)pl.box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(w), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    // one 32-byte load per neighbour slice when every slice start is 32-byte aligned
    const bool wide = s.Cin % 16 == 0 && s.Cg % 16 == 0 && (reinterpret_cast<uintptr_t>(x) & 31) == 0;
    auto kernel = wide ? dcn_fwd_tc_kernel<true> : dcn_fwd_tc_kernel<false>;
    static DeviceFlags attr_set[2];
    static DeviceCarveout carve[2];
    cudaError_t e = max_dynamic_smem_once((const void*)kernel, 227 * 1024, attr_set[wide]);
    if (e != cudaSuccess) return e;
    e = smem_carveout_for((const void*)kernel, pl.smem_bytes, carve[wide]);
    if (e != cudaSuccess) return e;
    int* counters = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + pl.ws_counters_off);
    e = cudaMemsetAsync(counters, 0, (size_t)pl.tiles * sizeof(int), st);
    if (e != cudaSuccess) return e;
    FwdArgs a;
    a.s = s;
    a.x = (const bf16*)x;
    a.off = (const bf16*)off;
    a.mask = (const bf16*)mask;
    a.bias = (const bf16*)bias;
    a.y = (bf16*)y;
    a.partials = reinterpret_cast<float*>(ws);
    a.counters = counters;
    a.status = status;
    a.n_tiles = pl.n_tiles;
    a.tiles = pl.tiles;
    a.U = pl.U;
    a.nq = pl.nq;
    a.sw = pl.sw;
    a.nf = pl.nf;
    a.wl = pl.wl;
    a.ctas = pl.ctas;
    a.total_units = pl.total_units;
    a.snap = pl.snap;
    a.bn_total = pl.bn_total;
    a.nsub = pl.nsub;
    a.box_rows = pl.box_rows;
    a.stages = pl.stages;
    a.acc_cols = pl.acc_cols;
    a.tmem_cols = pl.tmem_cols;
    a.b_off = pl.b_off;
    a.info_off = pl.info_off;
    a.row_off = pl.row_off;
    a.bar_off = pl.bar_off;
    a.b_stage_bytes = pl.b_stage_bytes;
    kernel<<<pl.ctas, NUM_THREADS, pl.smem_bytes, st>>>(map, a);
    if (launches) *launches += 2;
    return cudaGetLastError();
}


// ------------------------------------------------- forward without allocation --
// Scratch for callers that cannot allocate device memory themselves (see
// dcn_forward_noalloc in include/dcn.h). The array lives in this module's
// device image, so every GPU that loads the library holds it until the
// process exits; all calls share it.
namespace {

constexpr size_t kStaticScratchBytes = 48ull << 20;  // 48 MiB
static __device__ __align__(256) unsigned char g_fwd_scratch[kStaticScratchBytes];

// Device address of g_fwd_scratch on the current device, looked up once per
// device. In host code the symbol itself is only a host-side handle, never a
// device address, so kernels must get this pointer instead.
cudaError_t static_scratch_ptr(void** out) {
    static void* cache[64] = {nullptr};
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!cache[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_fwd_scratch);
        if (e != cudaSuccess) return e;
        cache[dev] = p;
    }
    *out = cache[dev];
    return cudaSuccess;
}

}  // namespace

size_t fwd_tc_static_scratch_bytes() { return kStaticScratchBytes; }

cudaError_t fwd_tc_noalloc(const Shape& s, const void* x, const void* off, const void* mask, const void* w,
                           const void* bias, void* y, unsigned* status, cudaStream_t st, int* launches) {
    if (fwd_tc_workspace(s) > kStaticScratchBytes) return cudaErrorInvalidValue;
    void* scratch = nullptr;
    cudaError_t e = static_scratch_ptr(&scratch);
    if (e != cudaSuccess) return e;
    // fwd_tc clears the tile counters in the scratch before its kernel runs
    return fwd_tc(s, x, off, mask, w, bias, y, scratch, kStaticScratchBytes, status, st, launches);
}

}  // namespace dcn
