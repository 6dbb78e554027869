// Forward DCNv2 on sm_100a tensor cores, bfloat16 in / float32 accumulate, with
// the gathered operand in tensor memory (layers with Cout <= 256).
//
// Y[P x Cout] = Col[P x K*K*Cin] * W^T as in fwd_tc.cu (the im2col view of the
// deformable convolution: the "Deformable ConvNets" notes, im2col appendix and
// the y(p0) equations), but the producers write each gathered A chunk (128
// output pixels x 64 channels of one tap) into TMEM with tcgen05.st, and the
// MMA reads A from TMEM (tcgen05.mma ... [a-tmem], b-desc). The gathered tile
// never passes through shared memory: shared memory holds only the weight ring,
// the sampling records and the epilogue's staging, which leaves the rest of the
// SM's 256 KB to the L1 cache the gather hits in, and no shared-memory
// bandwidth goes to writing A or to the tensor cores reading it.
//
//   * 8 producer warps, two per TMEM lane quarter (a warp may only reach the
//     32 lanes of its index mod 4). Each warp owns 16 rows (pixels) of every
//     chunk; lane l gathers row (l / 4) and row (l / 4) + 8, 16 channels
//     (32 bytes) of each, l % 4 picking which 16 of the chunk's 64. The blended
//     rows go to TMEM with one tcgen05.st.16x256b.x4, whose fixed thread-to-
//     column map places channel c = 16j + 4n + e (j = l % 4) at K position
//     k = 16n + 4j + e of the chunk. The weights are read in that same order:
//     a pre-pass permutes W = [Cout, K*K*Cin] into the workspace as
//     W' = [Cout, units x 64], unit u's 64 columns in K order k (zero where the
//     group has no channel), so the product sums the same terms.
//   * 1 TMA warp loads the [N x 64] tiles of W' into a shared-memory ring.
//   * 1 MMA warp issues tcgen05.mma.kind::f16 (M=128, N=Cout tile, K=16) with A
//     from TMEM into a TMEM accumulator, and commits each stage's release.
//   * 4 epilogue warps build the sampling records one (tile, group) epoch ahead
//     and read the accumulator back (stream-K combine as in fwd_tc.cu).
//
// TMEM (512 columns): accumulators at column 0 (one of <= 256 columns, or two
// of <= 128), the A ring of 8 stages x 32 columns at column 256.
#include "fwd_common.cuh"

namespace dcn {
namespace {

constexpr int NUM_PROD_WARPS = 8;
constexpr int TMA_WARP = 4, MMA_WARP = 5, PROD_WARP0 = 6;  // warps 0-3: records and epilogue
constexpr int NUM_THREADS = (PROD_WARP0 + NUM_PROD_WARPS) * 32;
constexpr int A_STAGES = 8;                  // TMEM A ring
constexpr int A_COL = 256;                   // first TMEM column of the A ring
constexpr int A_STAGE_COLS = BK / 2;         // 64 bf16 per row = 32 columns
constexpr int MAX_B_STAGES = 4;
constexpr int SLICE_CH = 16;                 // channels one lane gathers per sample (32 bytes)
#ifndef DCN_FWD_TS_B_STAGES
#define DCN_FWD_TS_B_STAGES 3
#endif

// Sixteen 32-bit registers per thread into 16 TMEM lanes x 32 columns
// (16x256b shape, 4 repetitions): thread t writes lanes t/4 and t/4 + 8,
// columns 8n + 2(t%4) and 8n + 2(t%4) + 1 of repetition n.
__device__ __forceinline__ void tmem_st_16x256b_x4(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.16x256b.x4.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// D[tmem] (+)= A[tmem] * B[smem]^T, bf16 x bf16 -> f32 (A read from TMEM lanes 0..127).
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Records epochs: a layer with at most ALL_TAPS taps keeps all taps of one
// (tile, group) in a record buffer (one epoch = the group's nq * K*K chunks);
// a larger kernel (K = 6, 7) keeps one row of K taps (one epoch = K chunks).
constexpr int ALL_TAPS = 25;
constexpr int MAX_TAPS_TS = 49;
constexpr int TAP_TABLE = 64;  // entries of the shared-memory tap table

// Gather record of the transposed pass (MODE 1, the grad_x contraction): up
// to LIST_E (dY row, weight) entries of one (input pixel, tap), gathered in
// batches of four; entry e is read when bit e of vmask is set. The weights
// pair up as in TapRec, so the same packed blend sums each batch. (Eight
// entries in two batches halve the corners left to the atomic scatter but
// expose the second batch's load latency: slower overall on conv4.)
constexpr int LIST_E = 4;
struct __align__(16) ListRec {
    int p[LIST_E];  // dY rows: output pixels (b*Ho + ho)*Wo + wo whose sample reaches this pixel
    uint32_t w[LIST_E / 2];  // w[i]: lo = entry 2i's weight m * (corner weight), hi = entry 2i+1's (bf16)
    uint32_t vmask;
    uint32_t pad[LIST_E == 4 ? 1 : 3];
};
static_assert(sizeof(ListRec) == 8 * LIST_E, "ListRec: 16-byte multiple");

// r += the blend of four neighbour slices (as blend16, accumulating).
__device__ __forceinline__ void blend16_acc(uint32_t (&r)[8], const uint32_t (&v)[4][8], uint32_t w01_00,
                                            uint32_t w11_10) {
    const uint32_t w00 = __byte_perm(w01_00, 0, 0x1010), w01 = __byte_perm(w01_00, 0, 0x3232);
    const uint32_t w10 = __byte_perm(w11_10, 0, 0x1010), w11 = __byte_perm(w11_10, 0, 0x3232);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        asm("{\n\t"
            "fma.rn.bf16x2 %0, %1, %5, %0;\n\t"
            "fma.rn.bf16x2 %0, %2, %6, %0;\n\t"
            "fma.rn.bf16x2 %0, %3, %7, %0;\n\t"
            "fma.rn.bf16x2 %0, %4, %8, %0;\n\t}"
            : "+r"(r[q])
            : "r"(v[0][q]), "r"(v[1][q]), "r"(v[2][q]), "r"(v[3][q]), "r"(w00), "r"(w01), "r"(w10), "r"(w11));
    }
}

struct TsArgs {
    FwdArgs f;
    const uint8_t* recs;  // [m tiles][G][K*K][BM] records (workspace), tap-major: TapRec (MODE 0), ListRec (MODE 1)
    float* yf;            // MODE 1: float32 output, row pitch ldy, first column col0
    int ldy, col0;
    int ep_len, ep_taps;  // chunks per records epoch, taps held per record buffer
    int b_stages;
    int band_pf;          // MODE 0: prefetch each next tile's input rows into L2 (inputs that do not stay in L2)
    uint32_t idle_bytes;  // shared memory free after the last MMA (the weight ring)
};

// ------------------------------------------------------------ pre-pass --
// The pre-pass of a call. (1) W' [Cout][U*64] from W [Cout][K*K*Cin]: unit
// u = (g, q, tap) (taps innermost), K position k of the unit holds channel
// c = 16*((k >> 2) & 3) + 4*(k >> 4) + (k & 3) of chunk q of group g at tap
// `tap` (zero past the group's channels), one thread per 8 outputs (16 bytes);
// (2) the sampling record of every (m tile, group, tap, tile row), tap-major so
// that one (tile, group) epoch is one contiguous block; (3) the stream-K tile
// counters cleared. Blocks [0, wblocks) do (1) and (3), the rest (2).
__global__ void __launch_bounds__(256) dcn_fwd_prepass_kernel(const bf16* __restrict__ w, bf16* __restrict__ wp,
                                                              TapRec* __restrict__ recs, const FwdArgs a, int wblocks,
                                                              long long nrec) {
    const Shape& s = a.s;
    // the main kernel may be scheduled now; it waits for this grid's completion before reading its outputs
    asm volatile("griddepcontrol.launch_dependents;");
    // launched as a programmatic dependent of whatever the stream ran before (so that this grid's
    // launch overlaps its tail): nothing is read or written before that work is complete
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if ((int)blockIdx.x >= wblocks) {
        const long long r = (long long)(blockIdx.x - wblocks) * blockDim.x + threadIdx.x;
        if (r >= nrec) return;
        const int row = (int)(r % BM);
        const long long e = r / BM;  // (mt * G + g) * K2 + tap
        const int tp = (int)(e % s.K2);
        const long long mg = e / s.K2;
        recs[r] = record_at(a, (int)(mg / s.G), (int)(mg % s.G), row, tp);
        return;
    }
    const int nq = a.nq, U = a.U;
    const long long n8 = (long long)s.Cout * U * 8;
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < a.tiles) a.counters[i] = 0;
    if (i >= n8) return;
    const int k8 = (int)(i & 7);
    const long long ou = i >> 3;
    const int u = (int)(ou % U);
    const int o = (int)(ou / U);
    const int g = u / (nq * s.K2), q = (u / s.K2) % nq, tap = u % s.K2;
    uint2 v[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int kb = 2 * k8 + h;                  // 4-element block of k
        const int c = 16 * (kb & 3) + 4 * (kb >> 2);  // its first channel within the chunk
        const int cg = q * BK + c;
        v[h] = make_uint2(0u, 0u);
        if (cg < s.Cg)
            v[h] = *reinterpret_cast<const uint2*>(w + (size_t)o * s.KC + (size_t)tap * s.Cin + (size_t)g * s.Cg + cg);
    }
    *reinterpret_cast<uint4*>(wp + ((size_t)o * U + u) * BK + 8 * k8) = make_uint4(v[0].x, v[0].y, v[1].x, v[1].y);
}

// The input rows a tile's samples can reach (its output rows' taps plus a
// margin of BAND_MARGIN pixels for the offsets) into L2, one bulk prefetch per
// input row, so that the gather of a tile whose input has left L2 meets L2
// latency rather than DRAM latency. Issued for the next tile while the current
// one is gathered; samples beyond the margin are simply fetched when needed.
constexpr int BAND_MARGIN = 4;
__device__ __forceinline__ void prefetch_strip_part(const FwdArgs& a, int b, int ho_lo, int ho_hi, int wo_lo,
                                                    int wo_hi) {
    const Shape& s = a.s;
    const int reach = (s.K - 1) * s.dil + 1;
    const int y_lo = max(0, ho_lo * s.stride - s.pad - BAND_MARGIN);
    const int y_hi = min(s.H - 1, ho_hi * s.stride - s.pad + reach + BAND_MARGIN);
    const int x_lo = max(0, wo_lo * s.stride - s.pad - BAND_MARGIN);
    const int x_hi = min(s.W - 1, wo_hi * s.stride - s.pad + reach + BAND_MARGIN);
    if (y_lo > y_hi || x_lo > x_hi) return;
    const uint32_t bytes = (uint32_t)(x_hi - x_lo + 1) * (uint32_t)s.Cin * 2u;
    for (int y = y_lo; y <= y_hi; ++y)
        ptx::bulk_prefetch_l2(a.x + (((size_t)b * s.H + y) * s.W + x_lo) * s.Cin, bytes);
}
__device__ __forceinline__ void prefetch_tile_band(const FwdArgs& a, int t) {
    const Shape& s = a.s;
    const int mt = t / a.n_tiles;
    const int r0 = mt * BM, r1 = min(r0 + BM, s.P) - 1;
    const int p0 = strip_to_raster(r0, a), p1 = strip_to_raster(r1, a);
    if (p0 < 0 || p1 < 0) return;
    const int plane = s.Ho * s.Wo;
    const int b0 = p0 / plane, b1 = p1 / plane;
    const int ho0 = (p0 - b0 * plane) / s.Wo, wo0 = (p0 - b0 * plane) % s.Wo;
    const int ho1 = (p1 - b1 * plane) / s.Wo, wo1 = (p1 - b1 * plane) % s.Wo;
    const int st0 = min(wo0 / a.sw, a.nf), st1 = min(wo1 / a.sw, a.nf);  // strip index (nf: the narrow last one)
    auto strip_lo = [&](int st) { return st * a.sw; };
    auto strip_hi = [&](int st) { return st < a.nf ? st * a.sw + a.sw - 1 : s.Wo - 1; };
    if (b0 == b1 && st0 == st1) {
        prefetch_strip_part(a, b0, ho0, ho1, strip_lo(st0), strip_hi(st0));
    } else {  // the tile ends one strip (or image) and begins the next
        prefetch_strip_part(a, b0, ho0, s.Ho - 1, strip_lo(st0), strip_hi(st0));
        prefetch_strip_part(a, b1, 0, ho1, strip_lo(st1), strip_hi(st1));
    }
}

// Output column n0 of the tile's first row pointer, and the row pitch.
template <int MODE>
__device__ __forceinline__ auto out_col(const TsArgs& ta, int n0) {
    if constexpr (MODE == 0) return ta.f.y + n0;
    else return ta.yf + ta.col0 + n0;
}
template <int MODE>
__device__ __forceinline__ int out_ld(const TsArgs& ta) {
    return MODE == 0 ? ta.f.s.Cout : ta.ldy;
}

// --------------------------------------------------------------- kernel --
// WIDE: x is 32-byte aligned and Cin, Cg are multiples of 16, so a lane's
// 16-channel slice is one 32-byte load.
// MODE 0: the forward (Y = Col * W'^T, bf16 y + bias; bilinear TapRec records).
// MODE 1: the transposed pass of the backward (rows = input pixels, the
// gathered tensor is grad_y and the records are ListRec lists; float32 out).
template <bool WIDE, int MODE>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    dcn_fwd_ts_kernel(const __grid_constant__ CUtensorMap tmap_w, const TsArgs ta) {
    constexpr uint32_t REC_BYTES = MODE == 0 ? (uint32_t)sizeof(TapRec) : (uint32_t)sizeof(ListRec);
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const FwdArgs& a = ta.f;
    const Shape& s = a.s;

    uint8_t* sB = smem;  // weight ring: b_stages x [N x 128 B], 128-byte swizzle
    uint8_t* s_rec = smem + a.info_off;  // two buffers of BM * ep_taps records
    int2* s_tap = reinterpret_cast<int2*>(smem + a.row_off);        // per tap: (i*dil, j*dil)
    long long* s_starts = reinterpret_cast<long long*>(s_tap + TAP_TABLE);  // [ctas + 1] first unit of each CTA
    float* s_bias = reinterpret_cast<float*>(s_starts + MAX_CTAS + 2);  // [2][512] bias of a tile's columns
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + a.bar_off);
    uint64_t* a_full = bars;                      // [A_STAGES] every producer warp stored the chunk
    uint64_t* a_empty = a_full + A_STAGES;        // [A_STAGES] the MMAs reading the stage completed
    uint64_t* b_full = a_empty + A_STAGES;        // [MAX_B_STAGES] weight tile landed
    uint64_t* b_empty = b_full + MAX_B_STAGES;    // [MAX_B_STAGES] the MMAs reading it completed
    uint64_t* acc_full = b_empty + MAX_B_STAGES;  // [2]
    uint64_t* acc_empty = acc_full + 2;           // [2]
    uint64_t* drain = acc_empty + 2;
    uint64_t* tail_bar = drain + 1;               // bulk copy of other CTAs' partials for the last segment
    uint64_t* rec_full = tail_bar + 1;            // [2] an epoch's records copied in
    uint64_t* rec_empty = rec_full + 2;           // [2] every producer warp done with an epoch's records
    uint64_t* epi_bar = rec_empty + 2;
    uint64_t* fin_go = epi_bar + 1;  // the last segment's combine plan is known (producers may help)
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(fin_go + 1);
    volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
    volatile int* s_last = s_abort + 1;  // [2], by segment parity
    volatile int* s_help = s_last + 2;   // [2]: producers share the final combine; partials staged in smem

    if (threadIdx.x == 0) {
        for (int i = 0; i < A_STAGES; ++i) {
            ptx::mbar_init(ptx::smem_u32(&a_full[i]), NUM_PROD_WARPS);
            ptx::mbar_init(ptx::smem_u32(&a_empty[i]), 1);
        }
        for (int i = 0; i < MAX_B_STAGES; ++i) {
            ptx::mbar_init(ptx::smem_u32(&b_full[i]), 1);
            ptx::mbar_init(ptx::smem_u32(&b_empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(ptx::smem_u32(&acc_full[i]), 1);
            ptx::mbar_init(ptx::smem_u32(&acc_empty[i]), 4);
        }
        ptx::mbar_init(ptx::smem_u32(drain), 1);
        ptx::mbar_init(ptx::smem_u32(tail_bar), 1);
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(ptx::smem_u32(&rec_full[i]), 1);
            ptx::mbar_init(ptx::smem_u32(&rec_empty[i]), NUM_PROD_WARPS);
        }
        ptx::mbar_init(ptx::smem_u32(epi_bar), 4);
        ptx::mbar_init(ptx::smem_u32(fin_go), 1);
        *s_abort = 0;
        s_last[0] = s_last[1] = 0;
        s_help[0] = s_help[1] = 0;
        ptx::fence_mbar_init();
    }
    if (threadIdx.x < s.K2) {
        const int i = threadIdx.x / s.K;
        s_tap[threadIdx.x] = make_int2(i * s.dil, (threadIdx.x - i * s.K) * s.dil);
    }
    for (int c = threadIdx.x; c <= a.ctas; c += NUM_THREADS) s_starts[c] = unit_begin(c, a);
    if (warp == MMA_WARP) {
        ptx::tmem_alloc(ptx::smem_u32(s_tmem), 512u);
        ptx::tmem_relinquish();
    }
    if (warp == TMA_WARP && lane == 0) ptx::prefetch_tmap(&tmap_w);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *s_tmem;
    // Launched as a programmatic dependent of the pre-pass: everything above
    // (barriers, TMEM, the stream-K plan) overlapped its tail; the records, W'
    // and the tile counters it writes are read only after this point.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // MODE 1: the backward-data kernel that follows may start on the SMs this
    // grid leaves; it waits for this grid before it adds into grad_x, and what
    // it reads was complete before this point
    if constexpr (MODE == 1) asm volatile("griddepcontrol.launch_dependents;");

    const int cta = blockIdx.x;
    const long long ubeg = s_starts[cta], uend = s_starts[cta + 1];
    const SegList L = seg_list(ubeg, uend, a.U);
    if (warp >= PROD_WARP0) {
        // ------------------------------------------------------ producers --
        const int rb = 32 * (warp & 3) + 16 * ((warp - PROD_WARP0) >> 2);  // this warp's 16 TMEM lanes (rows)
        const int j4 = lane & 3;
        const int r0 = rb + (lane >> 2), r1 = r0 + 8;
        const uint32_t t_row = tmem_base + ((uint32_t)rb << 16) + (uint32_t)A_COL;
        const long long cin2 = (long long)s.Cin * 2, rp2 = (long long)s.W * cin2;
        const uint8_t* zb = reinterpret_cast<const uint8_t*>(g_zero_slice);
#ifdef DCN_CHECKED
        const size_t xbytes = (size_t)s.B * s.H * s.W * s.Cin * sizeof(bf16);  // range-checked build
#endif
        bool ok = true;
        // the first epoch's records (copied in by the epilogue side)
        if (L.ns > 0)
            ok = __all_sync(0xffffffffu, ptx::mbar_wait(ptx::smem_u32(&rec_full[0]), 0, s_abort, a.status, WAIT_LIMIT));
        int isi = 0, ik = 0, ik1 = 0, iepoch = 0;
        int ileft = 0, irb = 0;  // chunks left in the records epoch; first tap held by the record buffer
        Chunk ich{0, 0, 0};
        // shared-memory address of the current epoch's records: read with ld.shared,
        // which does not queue behind the gathers in the global-load path
        uint32_t irecs = ptx::smem_u32(s_rec);
        if (L.ns > 0) {
            const Seg s0 = seg_at(L, 0);
            ik = s0.k0;
            ik1 = s0.k1;
            ich = chunk_of(ik, a);
            ileft = ta.ep_len - ik % ta.ep_len;
            irb = ta.ep_taps == s.K2 ? 0 : ich.tap - ich.tap % s.K;
        }
        // loads of row `row` of the cursor chunk into v, its weights into w
        // batch: MODE 1's entries 4*batch .. 4*batch + 3
        auto issue = [&](uint32_t(&v)[4][8], uint32_t(&w)[2], int row, int batch = 0) {
            const int cg = ich.q * BK + j4 * SLICE_CH;
            const uint32_t cmask = cg < s.Cg ? 0xFu : 0u;
            const bool hi_ok = cg + 8 < s.Cg;  // upper 8 channels present (narrow loads only)
            const uint8_t* xc = reinterpret_cast<const uint8_t*>(a.x + ich.g * s.Cg + cg);
            const uint32_t ra = irecs + (uint32_t)((ich.tap - irb) * BM + row) * REC_BYTES;
            const uint8_t* pc[4];
            uint32_t vm;
            if constexpr (MODE == 0) {
                const uint4 rc = ptx::lds_v4(ra);
                w[0] = rc.x;  // TapRec::w01_00
                w[1] = rc.y;  // TapRec::w11_10
                vm = rc.w & cmask;  // TapRec::vmask
                const uint8_t* p = xc + (long long)(int)rc.z * cin2;  // TapRec::base
                pc[0] = p;
                pc[1] = p + cin2;
                pc[2] = p + rp2;
                pc[3] = p + rp2 + cin2;
            } else {
                const uint4 pe = ptx::lds_v4(ra + 16 * batch);  // ListRec::p of the batch
                if constexpr (LIST_E == 4) {
                    const uint4 rw = ptx::lds_v4(ra + 16);  // ListRec::w, vmask
                    w[0] = rw.x;
                    w[1] = rw.y;
                    vm = rw.z & cmask;
                } else {
                    const uint4 rw = ptx::lds_v4(ra + 4 * LIST_E);  // ListRec::w
                    const uint32_t vall = ptx::lds_v4(ra + 6 * LIST_E).x;  // ListRec::vmask
                    w[0] = batch ? rw.z : rw.x;
                    w[1] = batch ? rw.w : rw.y;
                    vm = (vall >> (4 * batch)) & cmask;
                }
                pc[0] = xc + (long long)(int)pe.x * cin2;
                pc[1] = xc + (long long)(int)pe.y * cin2;
                pc[2] = xc + (long long)(int)pe.z * cin2;
                pc[3] = xc + (long long)(int)pe.w * cin2;
            }
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
        auto advance = [&]() -> bool {
            ++ik;
            if (++ich.tap == s.K2) {
                ich.tap = 0;
                if (++ich.q == a.nq) {
                    ich.q = 0;
                    ++ich.g;
                }
            }
            bool new_epoch = --ileft == 0;
            if (ik == ik1) {
                const Seg sn = seg_at(L, ++isi);
                ik = sn.k0;
                ik1 = sn.k1;
                ich = chunk_of(ik, a);
                ileft = ta.ep_len - ik % ta.ep_len;
                new_epoch = true;
            } else if (new_epoch) {
                ileft = ta.ep_len;
            }
            if (new_epoch) {
                irb = ta.ep_taps == s.K2 ? 0 : ich.tap - ich.tap % s.K;
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&rec_empty[iepoch & 1]));
                ++iepoch;
                const int b = iepoch & 1;
                const uint32_t par = (uint32_t)(iepoch >> 1) & 1u;
                // warp-uniform outcome: the tcgen05.st below is warp-collective
                if (!__all_sync(0xffffffffu, ptx::mbar_wait(ptx::smem_u32(&rec_full[b]), par, s_abort, a.status,
                                                            WAIT_LIMIT)))
                    return false;
                irecs = ptx::smem_u32(s_rec + (size_t)b * BM * ta.ep_taps * REC_BYTES);
            }
            return true;
        };
        const long long total = uend - ubeg;  // chunks of this CTA
        uint32_t va[4][8], vb[4][8], wa[2], wb[2];
        if (ok && total > 0) {
            issue(va, wa, r0);
            issue(vb, wb, r1);
        }
        int stage = 0, prev = -1;
        uint32_t phase = 0;
        for (long long n = 0; n < total && ok; ++n) {
            if (!__all_sync(0xffffffffu, ptx::mbar_wait(ptx::smem_u32(&a_empty[stage]), phase ^ 1, s_abort, a.status,
                                                        WAIT_LIMIT))) {
                ok = false;
                break;
            }
            const bool more = n + 1 < total;
            uint32_t ta8[8], tb8[8];
            blend16(ta8, va, wa[0], wa[1]);
            if constexpr (MODE == 1 && LIST_E > 4) {
                // entries 4..7 of both rows of this chunk, then on to the next chunk
                issue(va, wa, r0, 1);
                blend16(tb8, vb, wb[0], wb[1]);
                issue(vb, wb, r1, 1);
                blend16_acc(ta8, va, wa[0], wa[1]);
            }
            if (more) {
                if (!advance()) {
                    ok = false;
                    break;
                }
                issue(va, wa, r0);
            }
            if constexpr (MODE == 1 && LIST_E > 4) blend16_acc(tb8, vb, wb[0], wb[1]);
            else blend16(tb8, vb, wb[0], wb[1]);
            if (more) issue(vb, wb, r1);
            uint32_t r[16];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                r[4 * m] = ta8[2 * m];
                r[4 * m + 1] = ta8[2 * m + 1];
                r[4 * m + 2] = tb8[2 * m];
                r[4 * m + 3] = tb8[2 * m + 1];
            }
            // the previous chunk's store has had this chunk's blend to land: publish it
            if (prev >= 0) {
                tmem_wait_st();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&a_full[prev]));
            }
            tmem_st_16x256b_x4(t_row + (uint32_t)(stage * A_STAGE_COLS), r);
            prev = stage;
            if (++stage == A_STAGES) {
                stage = 0;
                phase ^= 1;
            }
        }
        tmem_wait_st();
        if (ok && prev >= 0) {
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&a_full[prev]));
        }
        // The CTA's last segment: when this CTA finishes a shared tile there, the
        // three warps of each TMEM lane quarter (its epilogue warp and two
        // producers) split the combine of that tile by 64-column pairs.
        if (ok && L.ns > 0 &&
            __all_sync(0xffffffffu, ptx::mbar_wait(ptx::smem_u32(fin_go), 0, s_abort, a.status, WAIT_LIMIT)) &&
            s_help[0]) {
            const int seg = L.ns - 1;
            const Seg sg = seg_at(L, seg);
            const int t = sg.t;
            const int abuf = a.acc_cols ? (seg & 1) : 0;
            const uint32_t accph = a.acc_cols ? ((seg >> 1) & 1) : (seg & 1);
            const bool staged = s_help[1] != 0;
            const long long tu0 = (long long)t * a.U;
            const int c_lo = cta_of_unit(tu0, s_starts, a.ctas), c_hi = cta_of_unit(tu0 + a.U - 1, s_starts, a.ctas);
            const uint32_t tile_bytes = (uint32_t)BM * a.bn_total * 4;
            bool go = __all_sync(0xffffffffu, ptx::mbar_wait(ptx::smem_u32(&acc_full[abuf]), accph, s_abort, a.status,
                                                             WAIT_LIMIT));
            if (go && staged)
                go = __all_sync(0xffffffffu, ptx::mbar_wait(ptx::smem_u32(tail_bar), 0, s_abort, a.status, WAIT_LIMIT));
            if (go) {
                ptx::tc_fence_after();
                const int mt = t / a.n_tiles, n0 = (t % a.n_tiles) * a.bn_total;
                const int ncols = min(a.bn_total, s.Cout - n0);
                const int qd = warp & 3, role = 1 + ((warp - PROD_WARP0) >> 2);
                const int row = qd * 32 + lane;
                const int p = strip_to_raster(mt * BM + row, a);
                const uint32_t taddr = tmem_base + (uint32_t)(abuf * a.acc_cols) + ((uint32_t)(qd * 32) << 16);
                const float* sb = a.bias ? s_bias + (seg & 1) * 512 : nullptr;
                const uint32_t yoff = staged ? (uint32_t)(c_hi - c_lo) * tile_bytes : 0u;
                const uint32_t ybuf = (yoff + 12 * 4096 <= ta.idle_bytes)
                                          ? ptx::smem_u32(smem + yoff) + (uint32_t)(warp - PROD_WARP0 + 4) * 4096u
                                          : 0u;
                for (int pr2 = role; pr2 * 64 < ncols; pr2 += 3)
                    combine_rows(taddr, ncols, c_lo, c_hi, cta, staged, [&](int c) -> const float* {
                        if (staged)
                            return reinterpret_cast<const float*>(smem + (size_t)(c - c_lo - (c > cta)) * tile_bytes) + row * 4;
                        return partial_base(a, s_starts, c, tu0, row);
                    }, sb, ybuf, out_col<MODE>(ta, n0), p, out_ld<MODE>(ta), pr2 * 64, pr2 * 64 + 64);
            }
        }
    } else if (warp == TMA_WARP) {
        // ------------------------------------------------------- weights --
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued = 0, issued_par = 0;  // per stage: a load was issued / parity of the last one
            const uint32_t bytes = (uint32_t)(a.box_rows * BK * 2);
            bool ok = true;
            for (int si = 0; si < L.ns && ok; ++si) {
                const Seg sg = seg_at(L, si);
                const int n0 = (sg.t % a.n_tiles) * a.bn_total;
                for (int k = sg.k0; k < sg.k1; ++k) {
                    if (!ptx::mbar_wait(ptx::smem_u32(&b_empty[stage]), phase ^ 1, s_abort, a.status, WAIT_LIMIT)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = ptx::smem_u32(&b_full[stage]);
                    ptx::mbar_arrive_expect_tx(fb, bytes);
                    ptx::tma_load_2d(ptx::smem_u32(sB + stage * a.b_stage_bytes), &tmap_w, fb, k * BK, n0);
                    issued |= 1u << stage;
                    issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == ta.b_stages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            if (*s_abort) {
                // wait (bounded) for loads still in flight before shared memory is released
                volatile int dummy = 0;
                for (int i = 0; i < ta.b_stages; ++i)
                    if ((issued >> i) & 1u)
                        ptx::mbar_wait(ptx::smem_u32(&b_full[i]), (issued_par >> i) & 1u, &dummy, nullptr,
                                       WAIT_LIMIT);
            }
        }
        __syncwarp();
    } else if (warp == MMA_WARP) {
        // ----------------------------------------------------------- MMA --
        if (lane == 0) {
            int as = 0, bs = 0;
            uint32_t aph = 0, bph = 0;
            const uint32_t idesc = ptx::idesc_bf16_f32(BM, a.bn_total);
            const uint32_t b0 = ptx::smem_u32(sB);
            bool ok = true;
            for (int seg = 0; seg < L.ns && ok; ++seg) {
                const Seg sg = seg_at(L, seg);
                const int abuf = a.acc_cols ? (seg & 1) : 0;
                const uint32_t accph = a.acc_cols ? ((seg >> 1) & 1) : (seg & 1);
                if (!ptx::mbar_wait(ptx::smem_u32(&acc_empty[abuf]), accph ^ 1, s_abort, a.status, WAIT_LIMIT)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t d = tmem_base + (uint32_t)(abuf * a.acc_cols);
                for (int k = sg.k0; k < sg.k1; ++k) {
                    if (!ptx::mbar_wait(ptx::smem_u32(&a_full[as]), aph, s_abort, a.status, WAIT_LIMIT) ||
                        !ptx::mbar_wait(ptx::smem_u32(&b_full[bs]), bph, s_abort, a.status, WAIT_LIMIT)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t at = tmem_base + (uint32_t)(A_COL + as * A_STAGE_COLS);
                    const uint32_t bsm = b0 + bs * a.b_stage_bytes;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        mma_bf16_ts(d, at + kk * 8, ptx::sw128_desc(bsm + kk * 32), idesc,
                                    (k > sg.k0 || kk > 0) ? 1u : 0u);
                    ptx::mma_commit(ptx::smem_u32(&a_empty[as]));
                    ptx::mma_commit(ptx::smem_u32(&b_empty[bs]));
                    if (++as == A_STAGES) {
                        as = 0;
                        aph ^= 1;
                    }
                    if (++bs == ta.b_stages) {
                        bs = 0;
                        bph ^= 1;
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
        // As in fwd_tc.cu: the records are built one epoch ahead of the
        // producers in two buffers; building epoch e waits only for the
        // producers to release epoch e - 2, which needs no epilogue of this
        // segment, so the order cannot deadlock.
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const int per_g = a.nq * s.K2;  // chunks per group within a tile
        uint32_t ephase = 0;
        int rec_epoch = 0;
        int rseg = 0, rk = L.ns > 0 ? seg_at(L, 0).k0 : 0;
        bool ok = true;
        for (int seg = 0; seg < L.ns && ok; ++seg) {
            const Seg sg = seg_at(L, seg);
            const int t = sg.t;
            if constexpr (MODE == 0) {
                if (ta.band_pf && threadIdx.x == 0 && seg + 1 < L.ns) prefetch_tile_band(a, seg_at(L, seg + 1).t);
            }
            while (rseg < L.ns && (rseg <= seg || (rseg == seg + 1 && rk == seg_at(L, rseg).k0))) {
                const Seg rs = seg_at(L, rseg);
                const int b = rec_epoch & 1;
                const int re = rk / ta.ep_len;  // epoch within the tile
                const int rg = (re * ta.ep_len) / per_g, rt = ta.ep_taps == s.K2 ? 0 : ((re * ta.ep_len) % s.K2);
                if (threadIdx.x == 0) {
                    // buffer b is free once every producer warp has left epoch rec_epoch - 2
                    if (rec_epoch >= 2 && !ptx::mbar_wait(ptx::smem_u32(&rec_empty[b]), ((rec_epoch - 2) >> 1) & 1,
                                                          s_abort, a.status, WAIT_LIMIT)) {
                        ok = false;
                    } else {
                        ptx::fence_proxy_async_smem();  // the producers' reads before the copy's writes
                        const uint32_t bytes = (uint32_t)BM * ta.ep_taps * REC_BYTES;
                        const uint32_t fb = ptx::smem_u32(&rec_full[b]);
                        ptx::mbar_arrive_expect_tx(fb, bytes);
                        ptx::bulk_load(ptx::smem_u32(s_rec + (size_t)b * BM * ta.ep_taps * REC_BYTES),
                                       ta.recs + (((size_t)(rs.t / a.n_tiles) * s.G + rg) * s.K2 + rt) * BM * REC_BYTES,
                                       bytes, fb);
                    }
                }
                if (warp == 0) ok = __shfl_sync(0xffffffffu, ok, 0);  // warp 0 stays convergent
                if (!ok) break;
                rk = min((re + 1) * ta.ep_len, rs.k1);
                if (rk >= rs.k1 && ++rseg < L.ns) rk = seg_at(L, rseg).k0;
                ++rec_epoch;
            }
            if (!ok) break;

            const int abuf = a.acc_cols ? (seg & 1) : 0;
            const uint32_t accph = a.acc_cols ? ((seg >> 1) & 1) : (seg & 1);
            const bool full = (sg.k0 == 0 && sg.k1 == a.U);
            const bool last_proc = seg == L.ns - 1;  // the pipeline is idle after this segment's accumulator
            const long long tu0 = (long long)t * a.U;
            int c_lo = cta, c_hi = cta;
            if (!full) {
                c_lo = cta_of_unit(tu0, s_starts, a.ctas);
                c_hi = cta_of_unit(tu0 + a.U - 1, s_starts, a.ctas);
            }
            int cnt = -1;
            if (!full && threadIdx.x == 0) cnt = ptx::ld_relaxed_gpu(a.counters + t);
            if (!__all_sync(0xffffffffu, ptx::mbar_wait(ptx::smem_u32(&acc_full[abuf]), accph, s_abort, a.status,
                                                        WAIT_LIMIT))) {
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
            float* sbias = s_bias + (seg & 1) * 512;
            if (a.bias)
                for (int i = threadIdx.x; i < ncols; i += 4 * 32) sbias[i] = __bfloat162float(a.bias[n0 + i]);
            if (!epi_sync(epi_bar, ephase, s_abort, a.status)) {
                ok = false;
                break;
            }
            const float* sb = a.bias ? sbias : nullptr;
            const int p = strip_to_raster(mt * BM + row, a);
            const uint32_t taddr = tmem_base + (uint32_t)(abuf * a.acc_cols) + ((uint32_t)(quarter * 32) << 16);
            auto* ycol0 = out_col<MODE>(ta, n0);
            const int ldy = out_ld<MODE>(ta);
            if (s_last[seg & 1]) {
                const uint32_t tile_bytes = (uint32_t)BM * a.bn_total * 4;
                const bool staged = !full && last_proc && (uint32_t)(c_hi - c_lo) * tile_bytes <= ta.idle_bytes;
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
                    if (!__all_sync(0xffffffffu, ptx::mbar_wait(ptx::smem_u32(tail_bar), 0, s_abort, a.status,
                                                                WAIT_LIMIT))) {
                        ok = false;
                        break;
                    }
                }
                const uint32_t yoff = staged ? (uint32_t)(c_hi - c_lo) * tile_bytes : 0u;
                // in the last segment the producers take two thirds of the columns (64-column pairs)
                const bool help = last_proc && (ncols & 63) == 0 && yoff + 12 * 4096 <= ta.idle_bytes;
                if (last_proc && threadIdx.x == 0) {
                    s_help[1] = staged ? 1 : 0;
                    s_help[0] = help ? 1 : 0;
                    ptx::mbar_arrive(ptx::smem_u32(fin_go));
                }
                const uint32_t ybuf =
                    (last_proc && yoff + 4 * 4096 <= ta.idle_bytes) ? ptx::smem_u32(smem + yoff) + quarter * 4096 : 0u;
                auto part = [&](int c) -> const float* {
                    if (staged) return reinterpret_cast<const float*>(smem + (size_t)(c - c_lo - (c > cta)) * tile_bytes) + row * 4;
                    return partial_base(a, s_starts, c, tu0, row);
                };
                if (help) {
                    for (int pr2 = 0; pr2 * 64 < ncols; pr2 += 3)
                        combine_rows(taddr, ncols, c_lo, c_hi, cta, staged, part, sb, ybuf, ycol0, p, ldy, pr2 * 64,
                                     pr2 * 64 + 64);
                } else {
                    combine_rows(taddr, ncols, c_lo, c_hi, cta, staged, part, sb, ybuf, ycol0, p, ldy);
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&acc_empty[abuf]));
                if (!full && threadIdx.x == 0) a.counters[t] = 0;
            } else {
                if (last_proc && threadIdx.x == 0) {  // the producers have nothing to add here
                    s_help[0] = 0;
                    ptx::mbar_arrive(ptx::smem_u32(fin_go));
                }
                float* dst = const_cast<float*>(partial_base(a, s_starts, cta, tu0, row));
                tmem_rows<true>(taddr, a.bn_total, [&](uint32_t(&r)[32], int cc) {
                    float* b = dst + (size_t)(cc >> 5) * 8 * BM * 4;
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        *reinterpret_cast<uint4*>(b + q * BM * 4) = make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
                });
                // the accumulator is in the workspace now: hand it to the next segment's MMAs
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&acc_empty[abuf]));
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
                    // every contributor's partial, this CTA's included, is in the workspace
                    __threadfence();
                    combine_rows(taddr, ncols, c_lo, c_hi, cta, false, [&](int c) -> const float* {
                        return partial_base(a, s_starts, c, tu0, row);
                    }, sb, 0u, ycol0, p, ldy, 0, 1 << 30, true);
                    if (threadIdx.x == 0) a.counters[t] = 0;
                }
            }
        }
    }

    // ------------------------------------------------------------ teardown --
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, 512u);
    }
}

// ------------------------------------------------------------------- host --

struct TsPlan {
    bool ok;
    StreamK k;
    int bn_total, b_stages, acc_cols, ep_len, ep_taps;
    uint32_t b_stage_bytes, info_off, row_off, bar_off, smem_bytes, idle_bytes;
    size_t ws_partials, ws_counters_off, ws_wperm_off, ws_recs_off, ws_bytes;
    long long nrec;
};

// mode 0: the forward; mode 1: the transposed pass (ListRec records, kept
// outside this workspace).
TsPlan make_ts_plan(const Shape& s, int sms, int mode = 0) {
    TsPlan pl{};
    pl.ok = false;
    const uint32_t rec_bytes = mode ? (uint32_t)sizeof(ListRec) : (uint32_t)sizeof(TapRec);
    if (s.Cin % 8 || s.Cg % 8 || s.Cout % 8 || s.K2 > MAX_TAPS_TS || s.Cout > 256) return pl;
    pl.bn_total = (s.Cout + 31) / 32 * 32;
    pl.k = plan_stream_k(s, pl.bn_total, sms);
    // two accumulators of <= 128 columns, or one of <= 256, below the A ring at column 256
    pl.acc_cols = pl.bn_total <= 128 ? 128 : 0;
    pl.b_stage_bytes = (uint32_t)pl.bn_total * 128;
    pl.b_stages = std::min(DCN_FWD_TS_B_STAGES, MAX_B_STAGES);
    const uint32_t ring = (uint32_t)pl.b_stages * pl.b_stage_bytes;
    // all taps of a (tile, group) per record buffer when both buffers fit in 80 KB, else one kernel row
    const bool all_taps = s.K2 <= ALL_TAPS && 2u * BM * s.K2 * rec_bytes <= 80u * 1024u;
    pl.ep_taps = all_taps ? s.K2 : s.K;
    pl.ep_len = all_taps ? pl.k.nq * s.K2 : s.K;
    const uint32_t info_bytes = 2u * BM * (uint32_t)pl.ep_taps * rec_bytes;
    pl.info_off = ring;
    pl.row_off = pl.info_off + info_bytes;
    pl.bar_off = pl.row_off + (uint32_t)(TAP_TABLE * sizeof(int2) + (MAX_CTAS + 2) * sizeof(long long) +
                                         2 * 512 * sizeof(float));
    pl.smem_bytes = pl.bar_off + (2 * A_STAGES + 2 * MAX_B_STAGES + 17) * 8 + 32 + 1024;
    pl.idle_bytes = ring;
    if (pl.smem_bytes > 227 * 1024) return pl;
    pl.ws_partials = (size_t)pl.k.ctas * 2 * BM * pl.bn_total * sizeof(float);
    pl.ws_counters_off = (pl.ws_partials + 255) & ~(size_t)255;
    pl.ws_wperm_off = (pl.ws_counters_off + (size_t)pl.k.tiles * sizeof(int) + 255) & ~(size_t)255;
    pl.ws_recs_off = (pl.ws_wperm_off + (size_t)s.Cout * pl.k.U * BK * 2 + 255) & ~(size_t)255;
    pl.nrec = (long long)pl.k.m_tiles * s.G * s.K2 * BM;
    pl.ws_bytes = pl.ws_recs_off + (mode ? (size_t)0 : (size_t)pl.nrec * sizeof(TapRec));
    pl.ok = true;
    return pl;
}


// ------------------------------------------------- transposed pass (grad_x) --
// grad_x[q, g*Cg + c] = sum_tap sum_o H_g[q, tap, o] * w[o, tap, g*Cg + c], with
// H_g[q, tap, :] = the sum over the samples (p, corner n) of group g and tap
// whose bilinear neighbour n is input pixel q of m * (corner weight) * grad_y[p, :]
// (the transpose of the forward's sampling: the gradient equations of the
// "Deformable ConvNets" notes summed per input pixel instead of scattered).
// It runs as the main kernel above in MODE 1 on a virtual layer whose output
// pixels are the input pixels, whose gathered tensor is grad_y and whose
// output channels are one group's input channels.

// Row of input pixel q in the strip order of the virtual layer (the inverse of
// strip_to_raster for Ho = H, Wo = W).
__device__ __forceinline__ int raster_to_strip(int q, int H, int W, int sw, int nf, int wl) {
    const int plane = H * W;
    const int b = q / plane, rem = q - b * plane;
    const int y = rem / W, xx = rem - y * W;
    const int strip = xx / sw;
    if (strip < nf) return b * plane + strip * (H * sw) + y * sw + (xx - strip * sw);
    return b * plane + nf * H * sw + y * wl + (xx - nf * sw);
}

// One thread per (output pixel p, group-tap gt), for the sample's four corners
// n (their slot claims in flight together): a corner's key (p << 32 | n << 16
// | bf16 weight) takes the next slot of its input pixel's list (LIST_CAP
// slots; the count in cnt, zero on entry). A corner past the last slot is
// flagged in ovf[gt * ovf_pitch + p] (bit n, zero on entry); the pre-pass
// below sorts each list and keeps its LIST_E smallest keys, so the lists and
// the flagged corners do not depend on the order of the insertions. Corners
// outside the map or of zero (bf16) weight add nothing and are skipped. The
// thread also writes the sample's float32 record for the backward-data kernel
// (rec[gt * ovf_pitch + p]: fractions, mask, (y0 + 1) << 16 | (x0 + 1), or all
// bits set when no corner is inside).
constexpr int LIST_CAP = 2 * LIST_E;
__device__ __forceinline__ void gxt_fill(const Shape& s, const bf16* __restrict__ off, const bf16* __restrict__ mask,
                                         int* __restrict__ cnt, unsigned long long* __restrict__ keys,
                                         uint8_t* __restrict__ ovf, float4* __restrict__ rec, int ovf_pitch,
                                         int mtiles_v, int sw, int nf, int wl) {
    const int p = blockIdx.x * blockDim.x + threadIdx.x;
    const int gt = blockIdx.y;
    if (p >= s.P) return;
    const int g = gt / s.K2, tap = gt - g * s.K2;
    const int plane = s.Ho * s.Wo;
    const int b = p / plane, pix = p - b * plane;
    const int ho = pix / s.Wo, wo = pix - ho * s.Wo;
    const int i = tap / s.K, j = tap - i * s.K;
    const bf16* offp = off + ((size_t)b * 2 * s.G * s.K2 + (size_t)g * 2 * s.K2 + 2 * tap) * plane + pix;
    const float dy = __bfloat162float(offp[0]), dx = __bfloat162float(offp[plane]);
    const float mk = mask ? __bfloat162float(mask[((size_t)b * s.G * s.K2 + (size_t)g * s.K2 + tap) * plane + pix])
                          : 1.f;
    int y0, x0;
    float ly, lx;
    split_coord(ho * s.stride - s.pad + i * s.dil, dy, y0, ly);
    split_coord(wo * s.stride - s.pad + j * s.dil, dx, x0, lx);
    if (rec) {
        const bool any = inside(s, y0, x0) || inside(s, y0, x0 + 1) || inside(s, y0 + 1, x0) || inside(s, y0 + 1, x0 + 1);
        rec[(size_t)gt * ovf_pitch + p] =
            make_float4(ly, lx, mk, __uint_as_float(any ? (((uint32_t)(y0 + 1) << 16) | (uint32_t)(x0 + 1)) : 0xFFFFFFFFu));
    }
    size_t L[4];
    int slot[4];
    unsigned short wbs[4];
#pragma unroll
    for (int n = 0; n < 4; ++n) {
        slot[n] = -1;
        L[n] = 0;
        wbs[n] = 0;
        const int yy = y0 + (n >> 1), xx = x0 + (n & 1);
        if (!inside(s, yy, xx)) continue;
        const float wf = ((n >> 1) ? ly : 1.f - ly) * ((n & 1) ? lx : 1.f - lx) * mk;
        const unsigned short wb = __bfloat16_as_ushort(__float2bfloat16_rn(wf));
        if ((wb & 0x7FFFu) == 0) continue;
        const int sr = raster_to_strip((b * s.H + yy) * s.W + xx, s.H, s.W, sw, nf, wl);
        L[n] = ((size_t)(g * mtiles_v + sr / BM) * s.K2 + tap) * BM + (sr % BM);
        wbs[n] = wb;
        slot[n] = atomicAdd(cnt + L[n], 1);
    }
    unsigned flags = 0;
#pragma unroll
    for (int n = 0; n < 4; ++n) {
        if (slot[n] < 0) continue;
        if (slot[n] < LIST_CAP)
            keys[L[n] * LIST_CAP + slot[n]] = ((unsigned long long)p << 32) | ((unsigned long long)n << 16) | wbs[n];
        else
            flags |= 1u << n;
    }
    if (flags) {
        const size_t at = (size_t)gt * ovf_pitch + p;
        atomicOr(reinterpret_cast<unsigned*>(ovf + (at & ~(size_t)3)), flags << (8 * (at & 3)));
    }
}
__global__ void __launch_bounds__(256) dcn_gxt_fill_kernel(const Shape s, const bf16* __restrict__ off,
                                                           const bf16* __restrict__ mask, int* __restrict__ cnt,
                                                           unsigned long long* __restrict__ keys,
                                                           uint8_t* __restrict__ ovf, float4* __restrict__ rec,
                                                           int ovf_pitch, int mtiles_v, int sw, int nf, int wl) {
    // the pre-pass may start: its weight blocks do not read what this grid writes
    asm volatile("griddepcontrol.launch_dependents;");
    gxt_fill(s, off, mask, cnt, keys, ovf, rec, ovf_pitch, mtiles_v, sw, nf, wl);
    // launched as a programmatic dependent of the backward-data transpose (which writes nothing
    // this grid touches): this grid completes only after it, so that everything after the
    // pre-pass may take both as done
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Pre-pass of one group's launch. Blocks [0, wblocks): W' of the virtual layer,
// W'[c][u*64 + k] = w[o][tap][g*Cg + c] for unit u = (q, tap) (taps innermost)
// and o = 64 q + (16*((k >> 2) & 3) + 4*(k >> 4) + (k & 3)) (zero past Cout),
// the order the producers store a chunk in; and the stream-K counters cleared.
// The other blocks turn the group's lists into ListRec records: a list of at
// most LIST_CAP keys keeps its LIST_E smallest and flags the rest in ovf; a
// longer one (some of its keys were never stored) flags all it holds and keeps
// none, its other corners having flagged themselves.
__global__ void __launch_bounds__(256) dcn_gxt_prepass_kernel(const Shape s, const bf16* __restrict__ w,
                                                              bf16* __restrict__ wp, ListRec* __restrict__ lrecs,
                                                              const int* __restrict__ cnt,
                                                              const unsigned long long* __restrict__ keys,
                                                              uint8_t* __restrict__ ovf, int ovf_pitch,
                                                              const FwdArgs a, int g, int wblocks, long long nrec) {
    asm volatile("griddepcontrol.launch_dependents;");
    if ((int)blockIdx.x >= wblocks) {
        // the lists are complete once the fill grid is (launched as its programmatic dependent)
        asm volatile("griddepcontrol.wait;" ::: "memory");
        const long long r = (long long)(blockIdx.x - wblocks) * blockDim.x + threadIdx.x;
        if (r >= nrec) return;
        const int c = cnt[r];
        const int tap = (int)((r / BM) % s.K2);
        const size_t gt = (size_t)g * s.K2 + tap;
        unsigned long long k[LIST_CAP];
        const int m = c < LIST_CAP ? c : LIST_CAP;
#pragma unroll
        for (int e = 0; e < LIST_CAP; ++e) k[e] = e < m ? keys[r * LIST_CAP + e] : ~0ull;
        // ascending order (insertion sort over the fixed-size array)
#pragma unroll
        for (int e = 1; e < LIST_CAP; ++e)
#pragma unroll
            for (int f = e; f > 0; --f) {
                const unsigned long long lo = k[f - 1] < k[f] ? k[f - 1] : k[f];
                const unsigned long long hi = k[f - 1] < k[f] ? k[f] : k[f - 1];
                k[f - 1] = lo;
                k[f] = hi;
            }
        const int keep = c > LIST_CAP ? 0 : (c < LIST_E ? c : LIST_E);
#pragma unroll
        for (int e = 0; e < LIST_CAP; ++e) {
            if (e < keep || e >= m) continue;
            const size_t at = gt * ovf_pitch + (size_t)(k[e] >> 32);
            atomicOr(reinterpret_cast<unsigned*>(ovf + (at & ~(size_t)3)), (1u << ((k[e] >> 16) & 3u)) << (8 * (at & 3)));
        }
        ListRec R;
        uint32_t wv[LIST_E];
        R.vmask = 0u;
#pragma unroll
        for (int e = 0; e < LIST_E; ++e) {
            const bool v = e < keep;
            R.p[e] = v ? (int)(k[e] >> 32) : 0;
            wv[e] = v ? (uint32_t)(k[e] & 0xFFFFu) : 0u;
            R.vmask |= v ? 1u << e : 0u;
        }
#pragma unroll
        for (int e = 0; e < LIST_E / 2; ++e) R.w[e] = wv[2 * e] | (wv[2 * e + 1] << 16);
#pragma unroll
        for (int e = 0; e < (int)(sizeof(R.pad) / 4); ++e) R.pad[e] = 0u;
        lrecs[r] = R;
        return;
    }
    const int U = a.U;
    const long long n8 = (long long)s.Cg * U * 8;
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < a.tiles) a.counters[i] = 0;
    if (i >= n8) return;
    const int c = (int)(i % s.Cg);  // consecutive threads read consecutive channels of w
    const long long uk = i / s.Cg;
    const int k8 = (int)(uk & 7), u = (int)(uk >> 3);
    const int q = u / s.K2, tap = u - q * s.K2;
    uint32_t v[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        float e2[2];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const int k = 8 * k8 + 2 * h + t;
            const int o = q * BK + 16 * ((k >> 2) & 3) + 4 * (k >> 4) + (k & 3);
            e2[t] = o < s.Cout ? __bfloat162float(w[(size_t)o * s.KC + (size_t)tap * s.Cin + (size_t)g * s.Cg + c]) : 0.f;
        }
        v[h] = pack_bf16(e2[0], e2[1]);
    }
    *reinterpret_cast<uint4*>(wp + ((size_t)c * U + u) * BK + 8 * k8) = make_uint4(v[0], v[1], v[2], v[3]);
}

// The virtual layer of the transposed pass for one group of s.
Shape gxt_shape(const Shape& s) {
    Shape v = s;
    v.H = s.Ho;  // the gathered tensor: grad_y [B, Ho, Wo, Cout]
    v.W = s.Wo;
    v.Ho = s.H;  // rows: the input pixels
    v.Wo = s.W;
    v.Cin = s.Cout;
    v.Cg = s.Cout;
    v.G = 1;
    v.Cout = s.Cg;
    v.P = s.B * s.H * s.W;
    v.KC = s.K2 * s.Cout;
    return v;
}

struct GxtPlan {
    bool ok;
    Shape v;
    TsPlan ts;
    size_t lists, lrec_bytes, cnt_off, keys_off, ts_off, ws_bytes;
};

GxtPlan make_gxt_plan(const Shape& s, int sms) {
    GxtPlan gp{};
    gp.ok = false;
    if (s.Cg > 256 || s.Cg % 8 || s.Cout % 8 || (long long)s.B * s.H * s.W >= (1LL << 31) / 64) return gp;
    gp.v = gxt_shape(s);
    gp.ts = make_ts_plan(gp.v, sms, 1);
    if (!gp.ts.ok) return gp;
    gp.lists = (size_t)s.G * gp.ts.k.m_tiles * s.K2 * BM;
    gp.lrec_bytes = gp.lists * sizeof(ListRec);
    gp.cnt_off = (gp.lrec_bytes + 255) & ~(size_t)255;
    gp.keys_off = (gp.cnt_off + gp.lists * sizeof(int) + 255) & ~(size_t)255;
    gp.ts_off = (gp.keys_off + gp.lists * LIST_CAP * sizeof(unsigned long long) + 255) & ~(size_t)255;
    gp.ws_bytes = gp.ts_off + gp.ts.ws_bytes;
    gp.ok = true;
    return gp;
}

// The kernel arguments a plan fixes (tensors and records are set by the caller).
TsArgs make_ts_args(const TsPlan& pl, const Shape& s, void* ws, int* counters, unsigned* status) {
    TsArgs ta{};
    FwdArgs& a = ta.f;
    a = FwdArgs{};
    a.s = s;
    a.partials = reinterpret_cast<float*>(ws);
    a.counters = counters;
    a.status = status;
    a.n_tiles = pl.k.n_tiles;
    a.tiles = pl.k.tiles;
    a.U = pl.k.U;
    a.nq = pl.k.nq;
    a.sw = pl.k.sw;
    a.nf = pl.k.nf;
    a.wl = pl.k.wl;
    a.ctas = pl.k.ctas;
    a.total_units = pl.k.total_units;
    a.snap = pl.k.snap;
    a.bn_total = pl.bn_total;
    a.nsub = 1;
    a.box_rows = pl.bn_total;
    a.stages = A_STAGES;
    a.acc_cols = pl.acc_cols;
    a.tmem_cols = 512;
    a.b_off = 0;
    a.info_off = pl.info_off;
    a.row_off = pl.row_off;
    a.bar_off = pl.bar_off;
    a.b_stage_bytes = pl.b_stage_bytes;
    ta.b_stages = pl.b_stages;
    ta.idle_bytes = pl.idle_bytes;
    ta.ep_len = pl.ep_len;
    ta.ep_taps = pl.ep_taps;
    return ta;
}

// The weight tensor map of a plan: W' [Cout][U*64] bf16, boxes of 64 x bn_total, 128-byte swizzle.
bool encode_wperm(CUtensorMap* map, const TsPlan& pl, const Shape& s, const void* wperm) {
    auto encode = get_encode();
    if (!encode) return false;
    cuuint64_t dims[2] = {(cuuint64_t)pl.k.U * BK, (cuuint64_t)s.Cout};
    cuuint64_t strides[1] = {(cuuint64_t)pl.k.U * BK * 2};
    cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)pl.bn_total};
    cuuint32_t estr[2] = {1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(wperm), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Launches the main kernel as a programmatic dependent of the pre-pass just enqueued on st.
template <int MODE>
cudaError_t launch_ts(const TsPlan& pl, const CUtensorMap& map, const TsArgs& ta, bool wide, cudaStream_t st) {
    auto kernel = wide ? dcn_fwd_ts_kernel<true, MODE> : dcn_fwd_ts_kernel<false, MODE>;
    static DeviceFlags attr_set[2];
    static DeviceCarveout carve[2];
    cudaError_t e = max_dynamic_smem_once((const void*)kernel, 227 * 1024, attr_set[wide]);
    if (e != cudaSuccess) return e;
    // the gather hits in L1: give it everything the kernel's shared memory does not need
    e = smem_carveout_for((const void*)kernel, pl.smem_bytes, carve[wide]);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)pl.k.ctas);
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = pl.smem_bytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kernel, map, ta);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}
}  // namespace

bool fwd_ts_supported(const Shape& s) { return make_ts_plan(s, num_sms()).ok; }

size_t fwd_ts_workspace(const Shape& s) {
    const TsPlan pl = make_ts_plan(s, num_sms());
    return pl.ok ? pl.ws_bytes : 0;
}

cudaError_t fwd_ts(const Shape& s, const void* x, const void* off, const void* mask, const void* w, const void* bias,
                   void* y, void* ws, size_t ws_bytes, unsigned* status, cudaStream_t st, int* launches) {
    const TsPlan pl = make_ts_plan(s, num_sms());
    if (!pl.ok || ws_bytes < pl.ws_bytes || !ws) return cudaErrorInvalidValue;
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    int* counters = reinterpret_cast<int*>(wsb + pl.ws_counters_off);
    bf16* wperm = reinterpret_cast<bf16*>(wsb + pl.ws_wperm_off);
    CUtensorMap map;
    if (!encode_wperm(&map, pl, s, wperm)) return cudaErrorInvalidValue;
    const bool wide = s.Cin % 16 == 0 && s.Cg % 16 == 0 && (reinterpret_cast<uintptr_t>(x) & 31) == 0;
    TsArgs ta = make_ts_args(pl, s, ws, counters, status);
    FwdArgs& a = ta.f;
    a.x = (const bf16*)x;
    a.off = (const bf16*)off;
    a.mask = (const bf16*)mask;
    a.bias = (const bf16*)bias;
    a.y = (bf16*)y;
    TapRec* recs = reinterpret_cast<TapRec*>(wsb + pl.ws_recs_off);
    ta.recs = reinterpret_cast<const uint8_t*>(recs);
    ta.yf = nullptr;
    ta.ldy = s.Cout;
    ta.col0 = 0;
    // an input of 64 MB or more does not stay in the 126 MB L2 between its tiles' gathers
    ta.band_pf = (size_t)s.B * s.H * s.W * s.Cin * sizeof(bf16) >= ((size_t)64 << 20) ? 1 : 0;
    const long long nw = std::max<long long>((long long)s.Cout * pl.k.U * 8, pl.k.tiles);
    const int wblocks = (int)((nw + 255) / 256);
    const long long rblocks = (pl.nrec + 255) / 256;
    cudaError_t e;
    {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(wblocks + rblocks));
        cfg.blockDim = dim3(256);
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, dcn_fwd_prepass_kernel, (const bf16*)w, wperm, recs, (const FwdArgs)a, wblocks,
                               pl.nrec);
        if (e != cudaSuccess) return e;
    }
    e = launch_ts<0>(pl, map, ta, wide, st);
    if (e != cudaSuccess) return e;
    if (launches) *launches += 2;
    return cudaSuccess;
}

bool gxt_supported(const Shape& s) { return make_gxt_plan(s, num_sms()).ok; }

cudaError_t gxt_prepare(const Shape& s, uint8_t* ovf, int ovf_pitch, void* ws, size_t ws_bytes, cudaStream_t st,
                        int* launches) {
    const GxtPlan gp = make_gxt_plan(s, num_sms());
    if (!gp.ok || !ws || ws_bytes < gp.ws_bytes || ovf_pitch < s.P) return cudaErrorInvalidValue;
    cudaError_t e = cudaMemsetAsync(static_cast<uint8_t*>(ws) + gp.cnt_off, 0, gp.lists * sizeof(int), st);
    if (e != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(ovf, 0, (size_t)s.G * s.K2 * ovf_pitch, st)) != cudaSuccess) return e;
    if (launches) *launches += 2;
    return cudaSuccess;
}

size_t gxt_workspace(const Shape& s) {
    const GxtPlan gp = make_gxt_plan(s, num_sms());
    return gp.ok ? gp.ws_bytes : 0;
}

cudaError_t gxt(const Shape& s, const void* off, const void* mask, const void* w, const void* gy, float* gx,
                uint8_t* ovf, void* rec, int ovf_pitch, void* ws, size_t ws_bytes, unsigned* status, cudaStream_t st,
                int* launches) {
    const GxtPlan gp = make_gxt_plan(s, num_sms());
    if (!gp.ok || !ws || ws_bytes < gp.ws_bytes || ovf_pitch < s.P) return cudaErrorInvalidValue;
    const TsPlan& pl = gp.ts;
    const Shape& v = gp.v;
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    ListRec* lrecs = reinterpret_cast<ListRec*>(wsb);
    int* cnt = reinterpret_cast<int*>(wsb + gp.cnt_off);
    unsigned long long* keys = reinterpret_cast<unsigned long long*>(wsb + gp.keys_off);
    uint8_t* tws = wsb + gp.ts_off;
    int* counters = reinterpret_cast<int*>(tws + pl.ws_counters_off);
    bf16* wperm = reinterpret_cast<bf16*>(tws + pl.ws_wperm_off);
    CUtensorMap map;
    if (!encode_wperm(&map, pl, v, wperm)) return cudaErrorInvalidValue;
    cudaError_t e;
    {
        // a programmatic dependent of the kernel before it (the caller's transpose of W, which
        // neither reads nor writes what the fill does); the counts and flags were zeroed by gxt_prepare
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)((s.P + 255) / 256), (unsigned)(s.G * s.K2));
        cfg.blockDim = dim3(256);
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, dcn_gxt_fill_kernel, s, (const bf16*)off, (const bf16*)mask, cnt, keys, ovf,
                               static_cast<float4*>(rec), ovf_pitch, pl.k.m_tiles, pl.k.sw, pl.k.nf, pl.k.wl);
        if (e != cudaSuccess) return e;
    }
    const bool wide = v.Cin % 16 == 0 && (reinterpret_cast<uintptr_t>(gy) & 31) == 0;
    const long long per_g = (long long)pl.k.m_tiles * s.K2 * BM;
    const long long nw = std::max<long long>((long long)v.Cout * pl.k.U * 8, pl.k.tiles);
    const int wblocks = (int)((nw + 255) / 256);
    const long long rblocks = (per_g + 255) / 256;
    int n = 1;
    for (int g = 0; g < s.G; ++g) {
        TsArgs ta = make_ts_args(pl, v, tws, counters, status);
        ta.f.x = (const bf16*)gy;
        ta.recs = reinterpret_cast<const uint8_t*>(lrecs + g * per_g);
        ta.yf = gx;
        ta.ldy = s.Cin;
        ta.col0 = g * s.Cg;
        {
            // a programmatic dependent of the fill (group 0; later groups follow the previous main kernel,
            // which lets no dependent start early)
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3((unsigned)(wblocks + rblocks));
            cfg.blockDim = dim3(256);
            cfg.stream = st;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            attr[0].val.programmaticStreamSerializationAllowed = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            e = cudaLaunchKernelEx(&cfg, dcn_gxt_prepass_kernel, s, (const bf16*)w, wperm, lrecs + g * per_g,
                                   (const int*)(cnt + g * per_g), (const unsigned long long*)(keys + (size_t)g * per_g * LIST_CAP),
                                   ovf, ovf_pitch, ta.f, g, wblocks, per_g);
            if (e != cudaSuccess) return e;
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        if ((e = launch_ts<1>(pl, map, ta, wide, st)) != cudaSuccess) return e;
        n += 2;
    }
    if (launches) *launches += n;
    return cudaSuccess;
}

}  // namespace dcn
