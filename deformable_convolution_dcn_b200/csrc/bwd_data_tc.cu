// Data-side backward of DCNv2 on sm_100a tensor cores (bfloat16 in, float32
// gradients): in one pass, grad_x, grad_offset and grad_mask.
//
// The column gradient G[p, (tap, c)] = sum_o grad_y[p, o] * w[o, tap, c] (the
// transpose of the forward's contraction, the col2im side of the im2col view in
// the "Deformable ConvNets" notes) is computed on tcgen05 tensor cores into TMEM,
// 128 output pixels x 256 channels of one (group, tap) per unit, K = Cout:
//   A = grad_y [P, Cout]                 TMA, 128-byte swizzle, K-major
//   B = w^T [K*K*Cin, Cout] (transposed once per call into the workspace)
// G never reaches HBM. Eight epilogue warps (two per TMEM lane quarter, each on
// half of the 256 channels) read it back and, per pixel, tap and channel, load
// the four bilinear neighbours of the sample and
//   * scatter G * m * (neighbour weight) into grad_x with 16-byte vector atomics,
//   * accumulate m * G * d(sample)/dy and d/dx (the offset gradient of the
//     notes' gradient equation, taken through floor()) and G * sample (the mask
//     gradient), added into grad_offset / grad_mask with one atomic per value.
// grad_x, grad_offset and grad_mask are zeroed first. Units (pixel tile,
// group-tap block) are split evenly over one CTA per SM; the TMEM accumulator
// is double-buffered so the epilogue of one unit overlaps the MMAs of the next.
// All waits are bounded.
//
// A second epilogue (EPI = 1, layers whose channels per group are a multiple of
// 64) works per pixel instead of per channel: with
//   S_n = sum_c G[c] * x_n[c]   (n = the four bilinear neighbours),
// the mask gradient is sum_n w_n S_n and the offset gradients are m times the
// differences of the S_n weighted by the other coordinate's fractions, so each
// (pixel, channel) costs four multiply-adds. W^T's rows are permuted so that the
// 16x256b TMEM load hands each thread 16 contiguous channels of two pixels,
// which are also one 32-byte load of each neighbour; no shared-memory
// transpose. grad_x is scattered from here only for the neighbours flagged in
// `ovf` (or all of them when no flags are given).
#include <cudaTypedefs.h>

#include <mutex>

#include "kernels.h"
#include "tc_ptx.cuh"

namespace dcn {
namespace {

constexpr int BM = 128;     // pixels per unit (UMMA M)
constexpr int NT = 256;     // channels per unit (UMMA N)
constexpr int BK = 64;      // output channels per K chunk
constexpr int EPI_WARPS = 8;
constexpr int TMA_WARP = 8, MMA_WARP = 9;
constexpr int NUM_THREADS = 10 * 32;
constexpr long long WAIT_LIMIT = 2000000000LL;
constexpr int MAX_STAGES = 4;
constexpr uint32_t A_BYTES = BM * BK * 2;   // 16 KB
constexpr uint32_t B_BYTES = NT * BK * 2;   // 32 KB
constexpr int TPITCH = 36;                  // floats per row of an epilogue warp's 32x32 transpose buffer
// grad_x through bwd_gx_tc.cu's shared-memory window (1) or this file's
// per-sample vector atomics (0, faster on the shapes measured so far)
#ifndef DCN_BWD_GX_WINDOW
#define DCN_BWD_GX_WINDOW 0
#endif
#ifndef DCN_BD_EPI1_STAGES
#define DCN_BD_EPI1_STAGES 2
#endif

struct BdArgs {
    Shape s;
    const bf16* x;
    const float4* rec;   // [G*K2][Ppad]: {ly, lx, m, ((y0+1) << 16) | (x0+1)} or yx = ~0 when all neighbours are outside
    float* gx;
    float* goff;
    float* gmask;
    const uint8_t* ovf;  // EPI 1: [G*K2][Ppad] neighbours (bit n) whose grad_x share is scattered here; null: all
    unsigned* status;
    int nblk, units_per_tile, m_tiles, ppad, ctas, stages, kchunks;
    long long total_units;
};

// 32 zero bytes: the source of every neighbour load that is not made (EPI 1).
__device__ __align__(32) uint32_t g_bd_zero[8];

// 16 TMEM lanes x 64 f32 columns from lane base `taddr` (16x256b shape, 8
// repetitions): for repetition m, registers 4m and 4m+1 hold lane t/4, columns
// 8m + 2(t%4) and 8m + 2(t%4) + 1, registers 4m+2 and 4m+3 lane t/4 + 8, the
// same columns (t: the thread's lane in the warp). Valid after tmem_wait_ld.
__device__ __forceinline__ void tmem_ld_16x256b_x8(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x8.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

// MMA column k (0..63) of a 64-channel block holds channel perm64(k): the
// 16x256b load then gives thread t%4 = j the channels 16j .. 16j + 15 in
// register-pair order (see tmem_ld_16x256b_x8). inv_perm64 is its inverse.
__host__ __device__ __forceinline__ int perm64(int k) { return 16 * ((k >> 1) & 3) + 2 * (k >> 3) + (k & 1); }
__host__ __device__ __forceinline__ int inv_perm64(int c) { return 8 * ((c >> 1) & 7) + 2 * (c >> 4) + (c & 1); }

__device__ __forceinline__ long long unit_begin(int c, const BdArgs& a) { return a.total_units * c / a.ctas; }

__device__ __forceinline__ float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

template <int EPI>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    dcn_bwd_data_tc_kernel(const __grid_constant__ CUtensorMap tmap_dy, const __grid_constant__ CUtensorMap tmap_wt,
                           const BdArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Shape& s = a.s;
    const uint32_t stage_bytes = A_BYTES + B_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + a.stages * stage_bytes);
    uint64_t* full = bars;
    uint64_t* empty = bars + MAX_STAGES;
    uint64_t* acc_full = bars + 2 * MAX_STAGES;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* drain = acc_empty + 2;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

    if (threadIdx.x == 0) {
        for (int i = 0; i < a.stages; ++i) {
            ptx::mbar_init(ptx::smem_u32(&full[i]), 1);
            ptx::mbar_init(ptx::smem_u32(&empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(ptx::smem_u32(&acc_full[i]), 1);
            ptx::mbar_init(ptx::smem_u32(&acc_empty[i]), EPI_WARPS);
        }
        ptx::mbar_init(ptx::smem_u32(drain), 1);
        *s_abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == MMA_WARP) {
        ptx::tmem_alloc(ptx::smem_u32(s_tmem), 512);
        ptx::tmem_relinquish();
    }
    if (warp == TMA_WARP && lane == 0) {
        ptx::prefetch_tmap(&tmap_dy);
        ptx::prefetch_tmap(&tmap_wt);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *s_tmem;
    const long long ubeg = unit_begin(blockIdx.x, a), uend = unit_begin(blockIdx.x + 1, a);

    if (warp == TMA_WARP) {
        // ------------------------------------------------- grad_y and w^T --
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, issued = 0, issued_par = 0;
            bool ok = true;
            for (long long u = ubeg; u < uend && ok; ++u) {
                const int mt = (int)(u / a.units_per_tile), r = (int)(u - (long long)mt * a.units_per_tile);
                const int gtap = r / a.nblk, cb = r - gtap * a.nblk;
                const int g = gtap / s.K2, tap = gtap - g * s.K2;
                const int row0 = tap * s.Cin + g * s.Cg + cb * NT;  // first w^T row (input channel) of the unit
                for (int kc = 0; kc < a.kchunks; ++kc) {
                    if (!ptx::mbar_wait(ptx::smem_u32(&empty[stage]), phase ^ 1, s_abort, a.status, WAIT_LIMIT)) {
                        ok = false;
                        break;
                    }
                    uint8_t* st = smem + stage * stage_bytes;
                    const uint32_t fb = ptx::smem_u32(&full[stage]);
                    ptx::mbar_arrive_expect_tx(fb, A_BYTES + B_BYTES);
                    ptx::tma_load_2d(ptx::smem_u32(st), &tmap_dy, fb, kc * BK, mt * BM);
                    ptx::tma_load_2d(ptx::smem_u32(st + A_BYTES), &tmap_wt, fb, kc * BK, row0);
                    issued |= 1u << stage;
                    issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == a.stages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            if (*s_abort) {
                volatile int dummy = 0;
                for (int i = 0; i < a.stages; ++i)
                    if ((issued >> i) & 1u)
                        ptx::mbar_wait(ptx::smem_u32(&full[i]), (issued_par >> i) & 1u, &dummy, nullptr, WAIT_LIMIT);
            }
        }
        __syncwarp();
    } else if (warp == MMA_WARP) {
        // ----------------------------------------------------------- MMA --
        if (lane == 0) {
            int stage = 0, seg = 0;
            uint32_t phase = 0;
            const uint32_t idesc = ptx::idesc_bf16_f32(BM, NT);
            const uint32_t s0 = ptx::smem_u32(smem);
            bool ok = true;
            for (long long u = ubeg; u < uend && ok; ++u, ++seg) {
                const int abuf = seg & 1;
                const uint32_t aphase = (seg >> 1) & 1;
                if (!ptx::mbar_wait(ptx::smem_u32(&acc_empty[abuf]), aphase ^ 1, s_abort, a.status, WAIT_LIMIT)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t d = tmem_base + (uint32_t)(abuf * NT);
                for (int kc = 0; kc < a.kchunks; ++kc) {
                    if (!ptx::mbar_wait(ptx::smem_u32(&full[stage]), phase, s_abort, a.status, WAIT_LIMIT)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t st = s0 + stage * stage_bytes;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        ptx::mma_bf16(d, ptx::sw128_desc(st + kk * 32), ptx::sw128_desc(st + A_BYTES + kk * 32), idesc,
                                      (kc > 0 || kk > 0) ? 1u : 0u);
                    ptx::mma_commit(ptx::smem_u32(&empty[stage]));
                    if (++stage == a.stages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                ptx::mma_commit(ptx::smem_u32(&acc_full[abuf]));
            }
            ptx::mma_commit(ptx::smem_u32(drain));
            volatile int dummy = 0;
            ptx::mbar_wait(ptx::smem_u32(drain), 0, &dummy, a.status, WAIT_LIMIT);
        }
        __syncwarp();
    } else if constexpr (EPI == 1) {
        // --------------------------------------------- per-pixel epilogue --
        // Warp w reads TMEM lanes rb .. rb + 15 (rb = 32 (w % 4) + 16 (w / 4));
        // thread t handles tile rows rb + t/4 and rb + t/4 + 8 and, in every
        // 64-column block, channels 16 (t % 4) .. + 15 of both.
        const int rbase = (warp & 3) * 32 + (warp >> 2) * 16;
        const int j = lane & 3;
        const int plane = s.Ho * s.Wo;
        const uint8_t* zb = reinterpret_cast<const uint8_t*>(g_bd_zero);
        const long long cin = s.Cin;
#ifdef DCN_CHECKED
        const size_t xbytes = (size_t)s.B * s.H * s.W * s.Cin * sizeof(bf16);  // range-checked build
        const size_t gxbytes = (size_t)s.B * s.H * s.W * s.Cin * sizeof(float);
#endif
        int seg = 0;
        bool ok = true;
        for (long long u = ubeg; u < uend && ok; ++u, ++seg) {
            const int abuf = seg & 1;
            const uint32_t aphase = (seg >> 1) & 1;
            const int mt = (int)(u / a.units_per_tile), r = (int)(u - (long long)mt * a.units_per_tile);
            const int gtap = r / a.nblk, cb = r - gtap * a.nblk;
            const int g = gtap / s.K2, tap = gtap - g * s.K2;
            const int c0 = cb * NT;
            const int nb64 = min(NT, s.Cg - c0) >> 6;  // 64-channel blocks of this unit (Cg % 64 == 0)
            // the two pixels' samples: fractions, mask, neighbours inside the map
            float4 rc[2];
            uint32_t fl[2], sc[2];
            long long q00[2];
            int pp[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int p = mt * BM + rbase + (lane >> 2) + 8 * h;
                pp[h] = p;
                rc[h] = make_float4(0.f, 0.f, 0.f, __uint_as_float(0xFFFFFFFFu));
                if (p < s.P) rc[h] = a.rec[(size_t)gtap * a.ppad + p];
                const uint32_t yx = __float_as_uint(rc[h].w);
                fl[h] = 0u;
                q00[h] = 0;
                if (p < s.P && yx != 0xFFFFFFFFu) {
                    const int y0 = (int)(yx >> 16) - 1, x0 = (int)(yx & 0xFFFFu) - 1;
                    fl[h] = (inside(s, y0, x0) ? 1u : 0u) | (inside(s, y0, x0 + 1) ? 2u : 0u) |
                            (inside(s, y0 + 1, x0) ? 4u : 0u) | (inside(s, y0 + 1, x0 + 1) ? 8u : 0u);
                    q00[h] = ((long long)(p / plane) * s.H + y0) * s.W + x0;
                }
                sc[h] = a.gx ? (a.ovf ? fl[h] & a.ovf[(size_t)gtap * a.ppad + min(p, a.ppad - 1)] : fl[h]) : 0u;
            }
            // neighbour n of pixel h: element offset (q00 + (n & 1) + (n >> 1) W) * Cin + this lane's channels
            const long long xoff = (long long)g * s.Cg + c0 + 16 * j;
            if (!__all_sync(0xffffffffu, ptx::mbar_wait(ptx::smem_u32(&acc_full[abuf]), aphase, s_abort, a.status,
                                                        WAIT_LIMIT))) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            const uint32_t tacc = tmem_base + (uint32_t)(abuf * NT) + ((uint32_t)rbase << 16);
            float S[2][4];
#pragma unroll
            for (int h = 0; h < 2; ++h) S[h][0] = S[h][1] = S[h][2] = S[h][3] = 0.f;
            for (int blk = 0; blk < nb64; ++blk) {
                uint32_t G[32];
                tmem_ld_16x256b_x8(tacc + (uint32_t)(blk * 64), G);
                uint32_t v[2][4][8];
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int n = 0; n < 4; ++n) {
                        const bf16* src = a.x + (q00[h] + (n & 1) + (n >> 1) * s.W) * cin + xoff + blk * 64;
#ifdef DCN_CHECKED
                        const bool rd = ((fl[h] >> n) & 1u) && ptx::in_range(src, 32, a.x, xbytes, a.status);
#else
                        const bool rd = (fl[h] >> n) & 1u;
#endif
                        ptx::ldg_v8(v[h][n], rd ? reinterpret_cast<const uint8_t*>(src) : zb);
                    }
                ptx::tmem_wait_ld(G);
                if (blk == nb64 - 1) {
                    // the accumulator is read: hand it to the MMAs of unit + 2
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&acc_empty[abuf]));
                }
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int n = 0; n < 4; ++n)
#pragma unroll
                        for (int m = 0; m < 8; ++m) {
                            S[h][n] = fmaf(__uint_as_float(G[4 * m + 2 * h]), bf_lo(v[h][n][m]), S[h][n]);
                            S[h][n] = fmaf(__uint_as_float(G[4 * m + 2 * h + 1]), bf_hi(v[h][n][m]), S[h][n]);
                        }
                if (sc[0] | sc[1]) {
                    // after the transposed pass has stored grad_x (a no-op unless launched as its dependent)
                    asm volatile("griddepcontrol.wait;" ::: "memory");
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const float ly = rc[h].x, lx = rc[h].y, mk = rc[h].z;
#pragma unroll
                        for (int n = 0; n < 4; ++n) {
                            if (!((sc[h] >> n) & 1u)) continue;
                            const float wy = (n >> 1) ? ly : 1.f - ly, wx = (n & 1) ? lx : 1.f - lx;
                            const float wnn = wy * wx * mk;
                            float* dst = a.gx + (q00[h] + (n & 1) + (n >> 1) * s.W) * cin + xoff + blk * 64;
#ifdef DCN_CHECKED
                            if (!ptx::in_range(dst, 64, a.gx, gxbytes, a.status)) continue;
#endif
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                ptx::red_add_v4(dst + 4 * i, __uint_as_float(G[8 * i + 2 * h]) * wnn,
                                                __uint_as_float(G[8 * i + 2 * h + 1]) * wnn,
                                                __uint_as_float(G[8 * i + 4 + 2 * h]) * wnn,
                                                __uint_as_float(G[8 * i + 5 + 2 * h]) * wnn);
                        }
                    }
                }
            }
            // S_n over the unit's channels: sum the four lanes of each pixel
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int n = 0; n < 4; ++n) {
                    S[h][n] += __shfl_xor_sync(0xffffffffu, S[h][n], 1);
                    S[h][n] += __shfl_xor_sync(0xffffffffu, S[h][n], 2);
                }
            if (j == 0) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int p = pp[h];
                    if (p >= s.P) continue;
                    const float ly = rc[h].x, lx = rc[h].y, mk = rc[h].z;
                    const float d_y = mk * ((1.f - lx) * (S[h][2] - S[h][0]) + lx * (S[h][3] - S[h][1]));
                    const float d_x = mk * ((1.f - ly) * (S[h][1] - S[h][0]) + ly * (S[h][3] - S[h][2]));
                    const float d_m = (1.f - ly) * ((1.f - lx) * S[h][0] + lx * S[h][1]) +
                                      ly * ((1.f - lx) * S[h][2] + lx * S[h][3]);
                    const int bb = p / plane, pix = p - bb * plane;
                    const size_t ob = ((size_t)bb * 2 * s.G * s.K2 + (size_t)g * 2 * s.K2 + 2 * tap) * plane + pix;
                    const size_t om = ((size_t)bb * s.G * s.K2 + (size_t)g * s.K2 + tap) * plane + pix;
                    if (a.nblk == 1) {  // this unit holds all of the group's channels: plain stores
                        if (a.goff) {
                            a.goff[ob] = d_y;
                            a.goff[ob + plane] = d_x;
                        }
                        if (a.gmask) a.gmask[om] = d_m;
                    } else {
                        if (a.goff) {
                            atomicAdd(a.goff + ob, d_y);
                            atomicAdd(a.goff + ob + plane, d_x);
                        }
                        if (a.gmask) atomicAdd(a.gmask + om, d_m);
                    }
                }
            }
        }
    } else {
        // ------------------------------------------------------ epilogue --
        // Thread = pixel row when reading TMEM; the 32x32 block of G is then
        // staged in shared memory and re-read so that 8 lanes cover one pixel's
        // 32 channels (4 each): neighbour loads are 64 contiguous bytes and the
        // grad_x atomics 128 contiguous bytes per pixel and corner.
        const int quarter = warp & 3, half = warp >> 2;  // lane quarter of TMEM, channel half
        const int row = quarter * 32 + lane;
        const int plane = s.Ho * s.Wo;
        float* tb = reinterpret_cast<float*>(smem + a.stages * stage_bytes + 1024) + warp * 32 * TPITCH;
        const int pq = lane >> 3, cj = lane & 7;  // pixel within a group of 4, 4-channel slot
#ifdef DCN_CHECKED
        const size_t xbytes = (size_t)s.B * s.H * s.W * s.Cin * sizeof(bf16);  // range-checked build
        const size_t gxbytes = (size_t)s.B * s.H * s.W * s.Cin * sizeof(float);
#endif
        int seg = 0;
        bool ok = true;
        for (long long u = ubeg; u < uend && ok; ++u, ++seg) {
            const int abuf = seg & 1;
            const uint32_t aphase = (seg >> 1) & 1;
            if (!ptx::mbar_wait(ptx::smem_u32(&acc_full[abuf]), aphase, s_abort, a.status, WAIT_LIMIT)) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            const int mt = (int)(u / a.units_per_tile), r = (int)(u - (long long)mt * a.units_per_tile);
            const int gtap = r / a.nblk, cb = r - gtap * a.nblk;
            const int g = gtap / s.K2, tap = gtap - g * s.K2;
            const int c_lo = cb * NT + half * (NT / 2);  // channel within the group
            const int nch = max(0, min(NT / 2, s.Cg - c_lo));
            const uint32_t taddr = tmem_base + (uint32_t)(abuf * NT + half * (NT / 2)) + ((uint32_t)(quarter * 32) << 16);
            // this thread's own pixel: sample and address of its top-left neighbour
            const int p = mt * BM + row;
            const float4 rc = (p < s.P) ? a.rec[(size_t)gtap * a.ppad + p] : make_float4(0.f, 0.f, 0.f, 0.f);
            const uint32_t yx = __float_as_uint(rc.w);
            const bool any = (p < s.P) && yx != 0xFFFFFFFFu;
            const int y0 = (int)(yx >> 16) - 1, x0 = (int)(yx & 0xFFFFu) - 1;
            const int b = p / plane;
            uint32_t flags = 0;
            if (any) {
                flags = (inside(s, y0, x0) ? 1u : 0u) | (inside(s, y0, x0 + 1) ? 2u : 0u) |
                        (inside(s, y0 + 1, x0) ? 4u : 0u) | (inside(s, y0 + 1, x0 + 1) ? 8u : 0u);
            }
            const long long a00 =
                any ? ((((long long)b * s.H + y0) * s.W + x0) * s.Cin + g * s.Cg + c_lo) : 0;
            float part[8][3];  // per pixel group: m-less d/dy, d/dx and the mask gradient, over this lane's channels
#pragma unroll
            for (int q = 0; q < 8; ++q) part[q][0] = part[q][1] = part[q][2] = 0.f;
            for (int cc = 0; cc < NT / 2; cc += 32) {
                float G[32];
                ptx::tmem_ld32(taddr + cc, G);
                if (cc >= nch) continue;  // warp-uniform
                __syncwarp();
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    *reinterpret_cast<float4*>(tb + lane * TPITCH + 4 * q) = make_float4(G[4 * q], G[4 * q + 1], G[4 * q + 2], G[4 * q + 3]);
                __syncwarp();
                const bool cv = cc + 4 * cj < nch;  // this lane's 4 channels inside the group
#pragma unroll
                for (int gp = 0; gp < 8; ++gp) {
                    const int src = 4 * gp + pq;  // lane (pixel row) whose sample this lane works on
                    const float ly = __shfl_sync(0xffffffffu, rc.x, src), lx = __shfl_sync(0xffffffffu, rc.y, src);
                    const float m = __shfl_sync(0xffffffffu, rc.z, src);
                    const uint32_t fl = __shfl_sync(0xffffffffu, flags, src);
                    const long long base = __shfl_sync(0xffffffffu, a00, src);
                    if (!fl || !cv) continue;
                    const float4 Gv = *reinterpret_cast<const float4*>(tb + src * TPITCH + 4 * cj);
                    const long long o00 = base + cc + 4 * cj;
                    const long long o01 = o00 + s.Cin, o10 = o00 + (long long)s.W * s.Cin, o11 = o10 + s.Cin;
#ifdef DCN_CHECKED
                    uint32_t flc = fl;
                    {
                        const long long oc[4] = {o00, o01, o10, o11};
                        for (int c = 0; c < 4; ++c)
                            if (((flc >> c) & 1u) &&
                                !(ptx::in_range(a.x + oc[c], 8, a.x, xbytes, a.status) &&
                                  (!a.gx || ptx::in_range(a.gx + oc[c], 16, a.gx, gxbytes, a.status))))
                                flc &= ~(1u << c);
                    }
#else
                    const uint32_t flc = fl;
#endif
                    const uint2 z = make_uint2(0, 0);
                    const uint2 v00 = (flc & 1u) ? ptx::ldg_v2(a.x + o00) : z;
                    const uint2 v01 = (flc & 2u) ? ptx::ldg_v2(a.x + o01) : z;
                    const uint2 v10 = (flc & 4u) ? ptx::ldg_v2(a.x + o10) : z;
                    const uint2 v11 = (flc & 8u) ? ptx::ldg_v2(a.x + o11) : z;
                    const float w00 = (1.f - ly) * (1.f - lx), w01 = (1.f - ly) * lx, w10 = ly * (1.f - lx), w11 = ly * lx;
                    const float Gc[4] = {Gv.x, Gv.y, Gv.z, Gv.w};
                    float r00[4], r01[4], r10[4], r11[4];
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const uint32_t wsel = h >> 1;
                        const uint32_t e00 = wsel ? v00.y : v00.x, e01 = wsel ? v01.y : v01.x;
                        const uint32_t e10 = wsel ? v10.y : v10.x, e11 = wsel ? v11.y : v11.x;
                        const float x00 = (h & 1) ? bf_hi(e00) : bf_lo(e00), x01 = (h & 1) ? bf_hi(e01) : bf_lo(e01);
                        const float x10 = (h & 1) ? bf_hi(e10) : bf_lo(e10), x11 = (h & 1) ? bf_hi(e11) : bf_lo(e11);
                        part[gp][2] = fmaf(Gc[h], w00 * x00 + w01 * x01 + w10 * x10 + w11 * x11, part[gp][2]);
                        part[gp][0] = fmaf(Gc[h], (1.f - lx) * (x10 - x00) + lx * (x11 - x01), part[gp][0]);
                        part[gp][1] = fmaf(Gc[h], (1.f - ly) * (x01 - x00) + ly * (x11 - x10), part[gp][1]);
                        const float gmc = Gc[h] * m;
                        r00[h] = gmc * w00;
                        r01[h] = gmc * w01;
                        r10[h] = gmc * w10;
                        r11[h] = gmc * w11;
                    }
                    if (a.gx) {
                        if (flc & 1u) ptx::red_add_v4(a.gx + o00, r00[0], r00[1], r00[2], r00[3]);
                        if (flc & 2u) ptx::red_add_v4(a.gx + o01, r01[0], r01[1], r01[2], r01[3]);
                        if (flc & 4u) ptx::red_add_v4(a.gx + o10, r10[0], r10[1], r10[2], r10[3]);
                        if (flc & 8u) ptx::red_add_v4(a.gx + o11, r11[0], r11[1], r11[2], r11[3]);
                    }
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&acc_empty[abuf]));
            // reduce each pixel's partial sums over its 8 lanes; lane cj == 0 adds them in
#pragma unroll
            for (int gp = 0; gp < 8; ++gp) {
#pragma unroll
                for (int k = 0; k < 3; ++k) {
                    float v = part[gp][k];
                    v += __shfl_xor_sync(0xffffffffu, v, 1);
                    v += __shfl_xor_sync(0xffffffffu, v, 2);
                    v += __shfl_xor_sync(0xffffffffu, v, 4);
                    part[gp][k] = v;
                }
                const int src = 4 * gp + pq;
                const float m = __shfl_sync(0xffffffffu, rc.z, src);
                const uint32_t fl = __shfl_sync(0xffffffffu, flags, src);
                const int pp = mt * BM + quarter * 32 + src;
                if (cj == 0 && fl && nch > 0 && pp < s.P) {
                    const int bb = pp / plane, pix = pp - bb * plane;
                    const size_t ob = ((size_t)bb * 2 * s.G * s.K2 + (size_t)g * 2 * s.K2 + 2 * tap) * plane + pix;
                    if (a.goff) {
                        atomicAdd(a.goff + ob, m * part[gp][0]);
                        atomicAdd(a.goff + ob + plane, m * part[gp][1]);
                    }
                    if (a.gmask)
                        atomicAdd(a.gmask + ((size_t)bb * s.G * s.K2 + (size_t)g * s.K2 + tap) * plane + pix, part[gp][2]);
                }
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, 512);
    }
}

// Float32 sampling records [G*K2][Ppad] for the backward: fractions, mask and
// the top-left neighbour (packed with +1 so that row/column -1 fits).
__global__ void __launch_bounds__(256) dcn_records_f32_kernel(Shape s, const bf16* __restrict__ off,
                                                              const bf16* __restrict__ mask, float4* __restrict__ rec,
                                                              int ppad) {
    const int p = blockIdx.x * blockDim.x + threadIdx.x;
    const int gt = blockIdx.y;
    if (p >= ppad) return;
    float4 r = make_float4(0.f, 0.f, 0.f, __uint_as_float(0xFFFFFFFFu));
    if (p < s.P) {
        const int g = gt / s.K2, tap = gt - g * s.K2;
        const TapSample t = tap_sample(s, off, mask, p, g, tap);
        const bool any = inside(s, t.y0, t.x0) || inside(s, t.y0, t.x0 + 1) || inside(s, t.y0 + 1, t.x0) ||
                         inside(s, t.y0 + 1, t.x0 + 1);
        r = make_float4(t.ly, t.lx, t.m,
                        __uint_as_float(any ? (((uint32_t)(t.y0 + 1) << 16) | (uint32_t)(t.x0 + 1)) : 0xFFFFFFFFu));
    }
    rec[(size_t)gt * ppad + p] = r;
}

// w [Cout, KC] -> wt [KC, Cout] (bf16), 32x32 tiles through shared memory.
// PERM: row k of wt goes to row (k & ~63) | inv_perm64(k & 63) (KC and the
// channel count a multiple of 64), the order the per-pixel epilogue reads.
template <bool PERM>
__global__ void __launch_bounds__(256) dcn_transpose_kernel(const bf16* __restrict__ w, bf16* __restrict__ wt,
                                                            int Cout, int KC) {
    // the transposed pass's fill may run alongside (it waits for this grid before it completes)
    asm volatile("griddepcontrol.launch_dependents;");
    __shared__ bf16 t[32][33];
    const int k0 = blockIdx.x * 32, o0 = blockIdx.y * 32;
    for (int i = threadIdx.y; i < 32; i += 8) {
        const int o = o0 + i, k = k0 + threadIdx.x;
        if (o < Cout && k < KC) t[i][threadIdx.x] = w[(size_t)o * KC + k];
    }
    __syncthreads();
    for (int i = threadIdx.y; i < 32; i += 8) {
        const int k = k0 + i, o = o0 + threadIdx.x;
        const int kd = PERM ? ((k & ~63) | inv_perm64(k & 63)) : k;
        if (o < Cout && k < KC) wt[(size_t)kd * Cout + o] = t[threadIdx.x][i];
    }
}

struct BdPlan {
    bool ok;
    int epi;  // 1: the per-pixel epilogue (channels per group a multiple of 64), else 0
    int nblk, units_per_tile, m_tiles, ppad, ctas, stages, kchunks;
    long long total_units;
    uint32_t smem_bytes;
    size_t rec_bytes, wt_off, ws_bytes;
    bool gxt;               // grad_x through the transposed gather-GEMM (per-pixel epilogue layers)
    size_t ovf_off, gxt_off;
};

// x32: x is 32-byte aligned (the per-pixel epilogue loads 32-byte slices)
BdPlan make_bd_plan(const Shape& s, int sms, bool x32 = true) {
    BdPlan pl{};
    if (s.Cin % 8 || s.Cg % 8 || s.Cout % 8 || s.H >= 65535 || s.W >= 65535) return pl;
    pl.nblk = (s.Cg + NT - 1) / NT;
    pl.units_per_tile = s.G * s.K2 * pl.nblk;
    pl.m_tiles = (s.P + BM - 1) / BM;
    pl.ppad = pl.m_tiles * BM;
    pl.kchunks = (s.Cout + BK - 1) / BK;
    pl.total_units = (long long)pl.m_tiles * pl.units_per_tile;
    pl.ctas = (int)std::min<long long>(sms, pl.total_units);
    pl.epi = (x32 && s.Cg % 64 == 0 && s.Cin % 64 == 0) ? 1 : 0;
    const uint32_t budget = 227 * 1024;
    const uint32_t tbytes = pl.epi ? 0u : (uint32_t)(EPI_WARPS * 32 * TPITCH * 4);  // epilogue transpose buffers
    int st = (int)((budget - 2048 - 1024 - tbytes) / (A_BYTES + B_BYTES));
    // the per-pixel epilogue's neighbour loads want L1 more than the MMAs want stages
    pl.stages = std::min(st, pl.epi ? DCN_BD_EPI1_STAGES : 3);
    pl.smem_bytes = pl.stages * (A_BYTES + B_BYTES) + 1024 + tbytes + 1024;
    pl.rec_bytes = (size_t)s.G * s.K2 * pl.ppad * sizeof(float4);
    pl.wt_off = (pl.rec_bytes + 255) & ~(size_t)255;
    pl.ws_bytes = pl.wt_off + (size_t)s.KC * s.Cout * sizeof(bf16);
    // grad_x without atomics where the transposed gather-GEMM takes the layer
    pl.gxt = pl.epi && gxt_supported(s);
    pl.ovf_off = pl.gxt_off = 0;
    if (pl.gxt) {
        pl.ovf_off = (pl.ws_bytes + 255) & ~(size_t)255;
        pl.gxt_off = (pl.ovf_off + (size_t)s.G * s.K2 * pl.ppad + 255) & ~(size_t)255;
        pl.ws_bytes = pl.gxt_off + gxt_workspace(s);
    }
    pl.ok = (long long)s.B * s.H * s.W * s.Cin < (1LL << 31);
    return pl;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

bool encode_kmajor(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
    auto encode = encode_fn();
    if (!encode) return false;
    cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)inner * 2};
    cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool bwd_data_tc_supported(const Shape& s) { return make_bd_plan(s, num_sms()).ok; }

size_t bwd_data_tc_workspace(const Shape& s) {
    BdPlan pl = make_bd_plan(s, num_sms());
    return pl.ok ? pl.ws_bytes : 0;
}

cudaError_t bwd_data_tc(const Shape& s, const void* x, const void* off, const void* mask, const void* w,
                        const void* gy, float* gx, float* goff, float* gmask, void* ws, size_t ws_bytes,
                        unsigned* status, cudaStream_t st, int* launches) {
    BdPlan pl = make_bd_plan(s, num_sms(), (reinterpret_cast<uintptr_t>(x) & 31) == 0);
    if (!pl.ok || !ws || ws_bytes < pl.ws_bytes) return cudaErrorInvalidValue;
    float4* rec = reinterpret_cast<float4*>(ws);
    bf16* wt = reinterpret_cast<bf16*>(static_cast<uint8_t*>(ws) + pl.wt_off);
    CUtensorMap map_dy, map_wt;
    if (!encode_kmajor(&map_dy, gy, (uint64_t)s.Cout, (uint64_t)s.P, BM) ||
        !encode_kmajor(&map_wt, wt, (uint64_t)s.Cout, (uint64_t)s.KC, NT))
        return cudaErrorInvalidValue;
    auto kernel = pl.epi ? dcn_bwd_data_tc_kernel<1> : dcn_bwd_data_tc_kernel<0>;
    static DeviceFlags attr_set[2];
    static DeviceCarveout carve[2];
    cudaError_t e = max_dynamic_smem_once((const void*)kernel, 227 * 1024, attr_set[pl.epi]);
    if (e != cudaSuccess) return e;
    // the rest of the SM's 256 KB is L1 for the neighbour loads
    e = smem_carveout_for((const void*)kernel, pl.smem_bytes, carve[pl.epi]);
    if (e != cudaSuccess) return e;
    int n = 0;
    if (gx && pl.gxt) {
        e = gxt_prepare(s, static_cast<uint8_t*>(ws) + pl.ovf_off, pl.ppad, static_cast<uint8_t*>(ws) + pl.gxt_off,
                        ws_bytes - pl.gxt_off, st, &n);
        if (e != cudaSuccess) return e;
    }
    dim3 tg((s.KC + 31) / 32, (s.Cout + 31) / 32);
    if (pl.epi) dcn_transpose_kernel<true><<<tg, dim3(32, 8), 0, st>>>((const bf16*)w, wt, s.Cout, s.KC);
    else dcn_transpose_kernel<false><<<tg, dim3(32, 8), 0, st>>>((const bf16*)w, wt, s.Cout, s.KC);
    ++n;
    // the sampling records: written by the transposed pass's fill kernel when it runs, else here
    if (!(gx && pl.gxt)) {
        dim3 rg((pl.ppad + 255) / 256, s.G * s.K2);
        dcn_records_f32_kernel<<<rg, 256, 0, st>>>(s, (const bf16*)off, (const bf16*)mask, rec, pl.ppad);
        ++n;
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // grad_x: the transposed gather-GEMM writes it (all but the flagged corners, which this
    // file's kernel then adds with atomics); otherwise zeroed here and scattered in full
    const uint8_t* ovf = nullptr;
    if (gx && pl.gxt) {
        uint8_t* ovf_w = static_cast<uint8_t*>(ws) + pl.ovf_off;
        e = gxt(s, off, mask, w, gy, gx, ovf_w, rec, pl.ppad, static_cast<uint8_t*>(ws) + pl.gxt_off,
                ws_bytes - pl.gxt_off, status, st, &n);
        if (e != cudaSuccess) return e;
        ovf = ovf_w;
    } else if (gx) {
        if ((e = cudaMemsetAsync(gx, 0, sizeof(float) * (size_t)s.B * s.H * s.W * s.Cin, st)) != cudaSuccess) return e;
        ++n;
    }
    // the per-pixel epilogue stores grad_offset / grad_mask outright when one unit holds a group's channels
    const bool zero_om = !(pl.epi && pl.nblk == 1);
    if (goff && zero_om) {
        if ((e = cudaMemsetAsync(goff, 0, sizeof(float) * (size_t)s.P * 2 * s.G * s.K2, st)) != cudaSuccess) return e;
        ++n;
    }
    if (gmask && zero_om) {
        if ((e = cudaMemsetAsync(gmask, 0, sizeof(float) * (size_t)s.P * s.G * s.K2, st)) != cudaSuccess) return e;
        ++n;
    }
    // grad_x through the shared-memory window kernel where it applies (and
    // DCN_BWD_GX_WINDOW is on); this file's kernel then computes only
    // grad_offset and grad_mask
    if (!pl.epi && DCN_BWD_GX_WINDOW && gx && bwd_gx_supported(s)) {
        e = bwd_gx_tc(s, gy, wt, rec, pl.ppad, gx, status, st, &n);
        if (e != cudaSuccess) return e;
        gx = nullptr;
        if (!goff && !gmask) {
            if (launches) *launches += n;
            return cudaSuccess;
        }
    }
    BdArgs a;
    a.s = s;
    a.x = (const bf16*)x;
    a.rec = rec;
    a.gx = gx;
    a.goff = goff;
    a.gmask = gmask;
    a.ovf = ovf;
    a.status = status;
    a.nblk = pl.nblk;
    a.units_per_tile = pl.units_per_tile;
    a.m_tiles = pl.m_tiles;
    a.ppad = pl.ppad;
    a.ctas = pl.ctas;
    a.stages = pl.stages;
    a.kchunks = pl.kchunks;
    a.total_units = pl.total_units;
    if (ovf) {
        // after the transposed pass: a programmatic dependent, whose CTAs start on the SMs that pass
        // frees and wait for it before their first grad_x atomic
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)pl.ctas);
        cfg.blockDim = dim3(NUM_THREADS);
        cfg.dynamicSmemBytes = pl.smem_bytes;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, kernel, map_dy, map_wt, a);
        if (e != cudaSuccess) return e;
    } else {
        kernel<<<pl.ctas, NUM_THREADS, pl.smem_bytes, st>>>(map_dy, map_wt, a);
    }
    ++n;
    if (launches) *launches += n;
    return cudaGetLastError();
}

}  // namespace dcn
