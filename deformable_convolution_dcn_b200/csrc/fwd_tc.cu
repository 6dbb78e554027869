// Forward DCNv2 on sm_100a tensor cores, bfloat16 in / float32 accumulate.
//
// The layer is the dense contraction Y[P x Cout] = Col[P x K*K*Cin] * W^T with
// P = B*Ho*Wo output pixels, where a row of Col holds the modulated bilinear
// samples m * x(p0 + p_k + dp_k) of one output pixel (the im2col view of the
// deformable convolution: the "Deformable ConvNets" notes, im2col appendix and
// the y(p0) equations). Col is never written to HBM:
//
//   * producer warps (8) compute the sampling coordinates of a 128-pixel tile,
//     load the four channel-contiguous NHWC neighbours of each sample as 16-byte
//     vectors, blend them with the bilinear weights times the mask, and store
//     the bf16 result straight into a shared-memory A tile laid out in the UMMA
//     128-byte-swizzle K-major canonical form;
//   * one TMA warp stages the matching weight tile [N x 64] of W = [Cout, K*K*Cin];
//   * one MMA warp issues tcgen05.mma (M=128, N<=256, K=16) into TMEM;
//   * four epilogue warps read the accumulator back with tcgen05.ld, add the
//     bias and store bf16 NHWC rows.
//
// The K loop runs over (group, 64-channel chunk, tap), taps innermost, so that
// consecutive chunks gather from the same 128-byte channel slice of nearby
// pixels while it is in L1. Work is split stream-K style: the (tile, chunk)
// units are divided evenly over one persistent CTA per SM; a tile that two or
// more CTAs share is summed from float32 partial tiles in the workspace by the
// CTA that finishes it last (counted with an atomic per tile; no CTA waits on
// another). Every wait is bounded and reports a timeout through the status word.
#include <cudaTypedefs.h>

#include <mutex>

#include "kernels.h"
#include "tc_ptx.cuh"

namespace dcn {
namespace {

constexpr int BM = 128;                 // output pixels per tile (UMMA M)
constexpr int BK = 64;                  // bf16 per K chunk (one 128-byte swizzle row)
constexpr int A_STAGE_BYTES = BM * BK * 2;
constexpr int NUM_PROD_WARPS = 8;
constexpr int TMA_WARP = 4, MMA_WARP = 5, PROD_WARP0 = 6;  // warps 0-3: epilogue
constexpr int NUM_THREADS = (PROD_WARP0 + NUM_PROD_WARPS) * 32;
constexpr int NUM_PROD_THREADS = NUM_PROD_WARPS * 32;
constexpr long long WAIT_LIMIT = 2000000000LL;  // clock cycles (about a second)
constexpr int MAX_STAGES = 8;

struct FwdArgs {
    Shape s;
    const bf16* x;
    const bf16* off;
    const bf16* mask;
    const bf16* bias;
    bf16* y;
    float* partials;   // [ctas][2][BM][bn_total]
    int* counters;     // [tiles], zero on entry
    unsigned* status;
    int n_tiles, tiles, U, nq, ctas;
    long long total_units;
    int bn_total;      // tile width in output channels (multiple of 16, <= 512)
    int nsub;          // accumulators per tile (1: N = bn_total; 2: 256 + rest)
    int box_rows;      // rows of one weight box
    int stages;
    int acc_cols;      // TMEM column stride between the two accumulator buffers (0: single buffer)
    int tmem_cols;
    uint32_t b_off, info_off, base_off, bar_off, b_stage_bytes;
};

__device__ __forceinline__ long long unit_begin(int c, const FwdArgs& a) {
    return a.total_units * c / a.ctas;
}
__device__ __forceinline__ int cta_of_unit(long long u, const FwdArgs& a) {
    return (int)(((u + 1) * a.ctas + a.total_units - 1) / a.total_units) - 1;
}

// Per-(row, tap) sampling record kept in shared memory for the current group:
// the four bilinear weights times the mask (zero for neighbours outside the
// map), as bf16 for the mixed-precision blend, and the pixel index of the
// top-left neighbour.
struct __align__(8) TapW {
    uint32_t w01_00;  // lo: w00, hi: w01
    uint32_t w11_10;  // lo: w10, hi: w11
};

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&t);
}

// acc[0..7] += w * (8 bf16 of v), f32 accumulation of bf16 products.
__device__ __forceinline__ void fma8(float (&acc)[8], const uint4& v, uint32_t wpair, bool hi_half) {
    uint16_t w = hi_half ? (uint16_t)(wpair >> 16) : (uint16_t)(wpair & 0xFFFFu);
    asm("{\n\t.reg .b16 a0, a1, a2, a3, a4, a5, a6, a7;\n\t"
        "mov.b32 {a0, a1}, %8;\n\t"
        "mov.b32 {a2, a3}, %9;\n\t"
        "mov.b32 {a4, a5}, %10;\n\t"
        "mov.b32 {a6, a7}, %11;\n\t"
        "fma.rn.f32.bf16 %0, a0, %12, %0;\n\t"
        "fma.rn.f32.bf16 %1, a1, %12, %1;\n\t"
        "fma.rn.f32.bf16 %2, a2, %12, %2;\n\t"
        "fma.rn.f32.bf16 %3, a3, %12, %3;\n\t"
        "fma.rn.f32.bf16 %4, a4, %12, %4;\n\t"
        "fma.rn.f32.bf16 %5, a5, %12, %5;\n\t"
        "fma.rn.f32.bf16 %6, a6, %12, %6;\n\t"
        "fma.rn.f32.bf16 %7, a7, %12, %7;\n\t}"
        : "+f"(acc[0]), "+f"(acc[1]), "+f"(acc[2]), "+f"(acc[3]), "+f"(acc[4]), "+f"(acc[5]), "+f"(acc[6]),
          "+f"(acc[7])
        : "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "h"(w));
}

// Tile t -> (m tile, n tile); chunk u -> (group, channel chunk, tap).
struct Chunk {
    int g, q, tap;
};
__device__ __forceinline__ Chunk chunk_of(int u, const FwdArgs& a) {
    Chunk c;
    int per_g = a.nq * a.s.K2;
    c.g = u / per_g;
    int r = u - c.g * per_g;
    c.q = r / a.s.K2;
    c.tap = r - c.q * a.s.K2;
    return c;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    dcn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmap_w, const FwdArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Shape& s = a.s;

    uint8_t* sA = smem;
    uint8_t* sB = smem + a.b_off;
    TapW* s_w = reinterpret_cast<TapW*>(smem + a.info_off);
    int* s_base = reinterpret_cast<int*>(smem + a.base_off);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + a.bar_off);
    // barrier slots
    uint64_t* full_a = bars;
    uint64_t* full_b = bars + MAX_STAGES;
    uint64_t* empty = bars + 2 * MAX_STAGES;
    uint64_t* acc_full = bars + 3 * MAX_STAGES;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* drain = acc_empty + 2;
    uint64_t* prod_bar = drain + 1;
    uint64_t* epi_bar = prod_bar + 1;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(epi_bar + 1);
    volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
    volatile int* s_last = s_abort + 1;

    if (threadIdx.x == 0) {
        for (int i = 0; i < a.stages; ++i) {
            ptx::mbar_init(ptx::smem_u32(&full_a[i]), NUM_PROD_WARPS);
            ptx::mbar_init(ptx::smem_u32(&full_b[i]), 1);
            ptx::mbar_init(ptx::smem_u32(&empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(ptx::smem_u32(&acc_full[i]), 1);
            ptx::mbar_init(ptx::smem_u32(&acc_empty[i]), 4);
        }
        ptx::mbar_init(ptx::smem_u32(drain), 1);
        ptx::mbar_init(ptx::smem_u32(prod_bar), NUM_PROD_WARPS);
        ptx::mbar_init(ptx::smem_u32(epi_bar), 4);
        *s_abort = 0;
        *s_last = 0;
        ptx::fence_mbar_init();
    }
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
    const long long ubeg = unit_begin(cta, a), uend = unit_begin(cta + 1, a);
    if (warp >= PROD_WARP0) {
        // ------------------------------------------------------ producers --
        const int ptid = threadIdx.x - PROD_WARP0 * 32;
        const int j = ptid & 7, r0 = ptid >> 3;
        int stage = 0;
        uint32_t phase = 0, pphase = 0;
        bool ok = true;
        for (long long u = ubeg; u < uend && ok;) {
            const int t = (int)(u / a.U);
            const int k0 = (int)(u - (long long)t * a.U);
            const int k1 = (int)min((long long)a.U, uend - (long long)t * a.U);
            const int mt = t / a.n_tiles;
            int cur_g = -1;
            for (int k = k0; k < k1 && ok; ++k) {
                const Chunk ch = chunk_of(k, a);
                if (ch.g != cur_g) {
                    // every producer is done with the previous records before they are overwritten
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(prod_bar));
                    if (!ptx::mbar_wait(ptx::smem_u32(prod_bar), pphase, s_abort, a.status, WAIT_LIMIT)) {
                        ok = false;
                        break;
                    }
                    pphase ^= 1;
                    for (int e = ptid; e < BM * s.K2; e += NUM_PROD_THREADS) {
                        const int tp = e / BM, row = e - tp * BM;
                        const int p = mt * BM + row;
                        float w00 = 0.f, w01 = 0.f, w10 = 0.f, w11 = 0.f;
                        int base = 0;
                        if (p < s.P) {
                            TapSample ts = tap_sample(s, a.off, a.mask, p, ch.g, tp);
                            const bool v00 = inside(s, ts.y0, ts.x0), v01 = inside(s, ts.y0, ts.x0 + 1);
                            const bool v10 = inside(s, ts.y0 + 1, ts.x0), v11 = inside(s, ts.y0 + 1, ts.x0 + 1);
                            w00 = v00 ? (1.f - ts.ly) * (1.f - ts.lx) * ts.m : 0.f;
                            w01 = v01 ? (1.f - ts.ly) * ts.lx * ts.m : 0.f;
                            w10 = v10 ? ts.ly * (1.f - ts.lx) * ts.m : 0.f;
                            w11 = v11 ? ts.ly * ts.lx * ts.m : 0.f;
                            if (v00 | v01 | v10 | v11) base = (ts.b * s.H + ts.y0) * s.W + ts.x0;
                        }
                        TapW tw;
                        tw.w01_00 = pack_bf16(w00, w01);
                        tw.w11_10 = pack_bf16(w10, w11);
                        s_w[row * s.K2 + tp] = tw;
                        s_base[row * s.K2 + tp] = base;
                    }
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(prod_bar));
                    if (!ptx::mbar_wait(ptx::smem_u32(prod_bar), pphase, s_abort, a.status, WAIT_LIMIT)) {
                        ok = false;
                        break;
                    }
                    pphase ^= 1;
                    cur_g = ch.g;
                }
                if (!ptx::mbar_wait(ptx::smem_u32(&empty[stage]), phase ^ 1, s_abort, a.status, WAIT_LIMIT)) {
                    ok = false;
                    break;
                }
                const int cg = ch.q * BK + j * 8;  // channel within the group
                const bool cval = cg < s.Cg;
                const bf16* xc = a.x + ch.g * s.Cg + cg;
                const long long rowpitch = (long long)s.W * s.Cin;
                uint4 v[4][4];
                TapW tw[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int row = r0 + 32 * i;
                    tw[i] = s_w[row * s.K2 + ch.tap];
                    const int base = s_base[row * s.K2 + ch.tap];
                    const bf16* pb = xc + (long long)base * s.Cin;
                    const uint4 z = make_uint4(0, 0, 0, 0);
                    v[i][0] = (cval && (tw[i].w01_00 & 0xFFFFu)) ? ptx::ldg_v4(pb) : z;
                    v[i][1] = (cval && (tw[i].w01_00 >> 16)) ? ptx::ldg_v4(pb + s.Cin) : z;
                    v[i][2] = (cval && (tw[i].w11_10 & 0xFFFFu)) ? ptx::ldg_v4(pb + rowpitch) : z;
                    v[i][3] = (cval && (tw[i].w11_10 >> 16)) ? ptx::ldg_v4(pb + rowpitch + s.Cin) : z;
                }
                const uint32_t a_stage = ptx::smem_u32(sA + stage * A_STAGE_BYTES);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int row = r0 + 32 * i;
                    float acc[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
                    fma8(acc, v[i][0], tw[i].w01_00, false);
                    fma8(acc, v[i][1], tw[i].w01_00, true);
                    fma8(acc, v[i][2], tw[i].w11_10, false);
                    fma8(acc, v[i][3], tw[i].w11_10, true);
                    uint4 o;
                    o.x = pack_bf16(acc[0], acc[1]);
                    o.y = pack_bf16(acc[2], acc[3]);
                    o.z = pack_bf16(acc[4], acc[5]);
                    o.w = pack_bf16(acc[6], acc[7]);
                    ptx::sts_v4(a_stage + row * 128 + ((j ^ (row & 7)) << 4), o);
                }
                ptx::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&full_a[stage]));
                if (++stage == a.stages) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            u = (long long)t * a.U + k1;
        }
    } else if (warp == TMA_WARP) {
        // ------------------------------------------------------- weights --
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued = 0, issued_par = 0;  // per stage: a load was issued / parity of the last one
            const uint32_t bytes = (uint32_t)(a.nsub * a.box_rows * BK * 2);
            bool ok = true;
            for (long long u = ubeg; u < uend && ok;) {
                const int t = (int)(u / a.U);
                const int k0 = (int)(u - (long long)t * a.U);
                const int k1 = (int)min((long long)a.U, uend - (long long)t * a.U);
                const int n0 = (t % a.n_tiles) * a.bn_total;
                for (int k = k0; k < k1; ++k) {
                    const Chunk ch = chunk_of(k, a);
                    if (!ptx::mbar_wait(ptx::smem_u32(&empty[stage]), phase ^ 1, s_abort, a.status, WAIT_LIMIT)) {
                        ok = false;
                        break;
                    }
                    const int xk = ch.tap * s.Cin + ch.g * s.Cg + ch.q * BK;
                    const uint32_t fb = ptx::smem_u32(&full_b[stage]);
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
                u = (long long)t * a.U + k1;
            }
            if (*s_abort) {
                // wait (bounded) for loads still in flight before shared memory is released
                volatile int dummy = 0;
                for (int i = 0; i < a.stages; ++i)
                    if ((issued >> i) & 1u)
                        ptx::mbar_wait(ptx::smem_u32(&full_b[i]), (issued_par >> i) & 1u, &dummy, nullptr,
                                       WAIT_LIMIT);
            }
        }
        __syncwarp();
    } else if (warp == MMA_WARP) {
        // ----------------------------------------------------------- MMA --
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int seg = 0;
            const uint32_t idesc0 = ptx::idesc_bf16_f32(BM, a.nsub == 1 ? a.bn_total : 256);
            const uint32_t idesc1 = ptx::idesc_bf16_f32(BM, a.nsub == 1 ? 16 : a.bn_total - 256);
            const uint32_t a0 = ptx::smem_u32(sA), b0 = ptx::smem_u32(sB);
            bool ok = true;
            for (long long u = ubeg; u < uend && ok; ++seg) {
                const int t = (int)(u / a.U);
                const int k0 = (int)(u - (long long)t * a.U);
                const int k1 = (int)min((long long)a.U, uend - (long long)t * a.U);
                const int abuf = a.acc_cols ? (seg & 1) : 0;
                const uint32_t aphase = a.acc_cols ? ((seg >> 1) & 1) : (seg & 1);
                if (!ptx::mbar_wait(ptx::smem_u32(&acc_empty[abuf]), aphase ^ 1, s_abort, a.status, WAIT_LIMIT)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t d = tmem_base + (uint32_t)(abuf * a.acc_cols);
                for (int k = k0; k < k1; ++k) {
                    if (!ptx::mbar_wait(ptx::smem_u32(&full_a[stage]), phase, s_abort, a.status, WAIT_LIMIT) ||
                        !ptx::mbar_wait(ptx::smem_u32(&full_b[stage]), phase, s_abort, a.status, WAIT_LIMIT)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t as = a0 + stage * A_STAGE_BYTES, bs = b0 + stage * a.b_stage_bytes;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint32_t acc = (k > k0 || kk > 0) ? 1u : 0u;
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
                u = (long long)t * a.U + k1;
            }
            // all MMAs issued by this thread complete before TMEM is released
            ptx::mma_commit(ptx::smem_u32(drain));
            volatile int dummy = 0;
            ptx::mbar_wait(ptx::smem_u32(drain), 0, &dummy, a.status, WAIT_LIMIT);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ epilogue --
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        int seg = 0;
        uint32_t ephase = 0;
        bool ok = true;
        for (long long u = ubeg; u < uend && ok; ++seg) {
            const int t = (int)(u / a.U);
            const int k0 = (int)(u - (long long)t * a.U);
            const int k1 = (int)min((long long)a.U, uend - (long long)t * a.U);
            const int abuf = a.acc_cols ? (seg & 1) : 0;
            const uint32_t aphase = a.acc_cols ? ((seg >> 1) & 1) : (seg & 1);
            if (!ptx::mbar_wait(ptx::smem_u32(&acc_full[abuf]), aphase, s_abort, a.status, WAIT_LIMIT)) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            const int mt = t / a.n_tiles, n0 = (t % a.n_tiles) * a.bn_total;
            const int p = mt * BM + row;
            const uint32_t taddr = tmem_base + (uint32_t)(abuf * a.acc_cols) + ((uint32_t)(quarter * 32) << 16);
            const bool full = (k0 == 0 && k1 == a.U);
            const int ncols = min(a.bn_total, s.Cout - n0);
            if (full) {
                bf16* yrow = a.y + (size_t)p * s.Cout + n0;
                for (int cc = 0; cc < a.bn_total; cc += 32) {
                    float v[32];
                    ptx::tmem_ld32(taddr + cc, v);
                    if (p < s.P && cc < ncols) {
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (a.bias && cc + e < ncols) v[e] += __bfloat162float(a.bias[n0 + cc + e]);
                        if (cc + 32 <= ncols) {
                            uint4* dst = reinterpret_cast<uint4*>(yrow + cc);
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                dst[q] = make_uint4(pack_bf16(v[8 * q], v[8 * q + 1]), pack_bf16(v[8 * q + 2], v[8 * q + 3]),
                                                    pack_bf16(v[8 * q + 4], v[8 * q + 5]),
                                                    pack_bf16(v[8 * q + 6], v[8 * q + 7]));
                        } else {
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                if (cc + e < ncols) yrow[cc + e] = __float2bfloat16_rn(v[e]);
                        }
                    }
                }
            } else {
                const int slot = (seg == 0) ? 0 : 1;
                float* dst = a.partials + (((size_t)cta * 2 + slot) * BM + row) * a.bn_total;
                for (int cc = 0; cc < a.bn_total; cc += 32) {
                    float v[32];
                    ptx::tmem_ld32(taddr + cc, v);
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        reinterpret_cast<float4*>(dst + cc)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&acc_empty[abuf]));
            if (!full) {
                __threadfence();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(epi_bar));
                if (!ptx::mbar_wait(ptx::smem_u32(epi_bar), ephase, s_abort, a.status, WAIT_LIMIT)) {
                    ok = false;
                    break;
                }
                ephase ^= 1;
                const long long tu0 = (long long)t * a.U, tu1 = tu0 + a.U;
                const int c_lo = cta_of_unit(tu0, a), c_hi = cta_of_unit(tu1 - 1, a);
                if (threadIdx.x == 0) {
                    const int old = atomicAdd(a.counters + t, 1);
                    *s_last = (old == c_hi - c_lo) ? 1 : 0;
                }
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(epi_bar));
                if (!ptx::mbar_wait(ptx::smem_u32(epi_bar), ephase, s_abort, a.status, WAIT_LIMIT)) {
                    ok = false;
                    break;
                }
                ephase ^= 1;
                if (*s_last) {
                    __threadfence();
                    if (p < s.P) {
                        bf16* yrow = a.y + (size_t)p * s.Cout + n0;
                        for (int cc = 0; cc < ncols; cc += 32) {
                            float v[32];
#pragma unroll
                            for (int e = 0; e < 32; ++e) v[e] = 0.f;
                            for (int c = c_lo; c <= c_hi; ++c) {
                                const int cslot = (unit_begin(c, a) >= tu0) ? 0 : 1;
                                const float* src = a.partials + (((size_t)c * 2 + cslot) * BM + row) * a.bn_total + cc;
#pragma unroll
                                for (int q = 0; q < 8; ++q) {
                                    float4 f = ptx::ldcg_f4(src + 4 * q);
                                    v[4 * q] += f.x;
                                    v[4 * q + 1] += f.y;
                                    v[4 * q + 2] += f.z;
                                    v[4 * q + 3] += f.w;
                                }
                            }
#pragma unroll
                            for (int e = 0; e < 32; ++e) {
                                if (cc + e < ncols) {
                                    float r = v[e] + (a.bias ? __bfloat162float(a.bias[n0 + cc + e]) : 0.f);
                                    yrow[cc + e] = __float2bfloat16_rn(r);
                                }
                            }
                        }
                    }
                    if (threadIdx.x == 0) a.counters[t] = 0;
                }
            }
            u = (long long)t * a.U + k1;
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
    long long total_units;
    uint32_t b_off, info_off, base_off, bar_off, b_stage_bytes, smem_bytes;
    size_t ws_partials, ws_counters_off, ws_bytes;
};

int num_sms() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

Plan make_plan(const Shape& s, int sms) {
    Plan pl{};
    pl.ok = false;
    if (s.Cin % 8 || s.Cg % 8 || s.Cout % 8 || s.K2 > 25) return pl;
    pl.bn_total = std::min(512, (s.Cout + 31) / 32 * 32);
    pl.n_tiles = (s.Cout + pl.bn_total - 1) / pl.bn_total;
    pl.m_tiles = (s.P + BM - 1) / BM;
    pl.tiles = pl.m_tiles * pl.n_tiles;
    pl.nq = (s.Cg + BK - 1) / BK;
    pl.U = s.G * pl.nq * s.K2;
    pl.total_units = (long long)pl.tiles * pl.U;
    pl.ctas = (int)std::min<long long>(sms, pl.total_units);
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
    const uint32_t info_bytes = (uint32_t)(BM * s.K2 * (sizeof(TapW) + sizeof(int)));
    const uint32_t fixed = info_bytes + 64 * 8 + 64 + 1024;  // info, barriers, flags, alignment slack
    const uint32_t budget = 227 * 1024;
    const uint32_t stage_bytes = A_STAGE_BYTES + pl.b_stage_bytes;
    int st = (int)((budget - fixed) / stage_bytes);
    st = std::min(st, 4);
    if (st < 2) return pl;
    pl.stages = st;
    pl.b_off = (uint32_t)(st * A_STAGE_BYTES);
    pl.info_off = pl.b_off + (uint32_t)st * pl.b_stage_bytes;
    pl.base_off = pl.info_off + (uint32_t)(BM * s.K2 * sizeof(TapW));
    pl.bar_off = (pl.base_off + (uint32_t)(BM * s.K2 * sizeof(int)) + 7) & ~7u;
    pl.smem_bytes = pl.bar_off + (3 * MAX_STAGES + 8) * 8 + 16 + 1024;
    if (pl.smem_bytes > budget) return pl;
    pl.ws_partials = (size_t)pl.ctas * 2 * BM * pl.bn_total * sizeof(float);
    pl.ws_counters_off = (pl.ws_partials + 255) & ~(size_t)255;
    pl.ws_bytes = pl.ws_counters_off + (size_t)pl.tiles * sizeof(int);
    pl.ok = true;
    return pl;
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
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

}  // namespace

bool fwd_tc_supported(const Shape& s) { return make_plan(s, num_sms()).ok; }

size_t fwd_tc_workspace(const Shape& s) {
    Plan pl = make_plan(s, num_sms());
    return pl.ok ? pl.ws_bytes : 0;
}

cudaError_t fwd_tc(const Shape& s, const void* x, const void* off, const void* mask, const void* w, const void* bias,
                   void* y, void* ws, size_t ws_bytes, unsigned* status, cudaStream_t st, int* launches) {
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
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        e = cudaFuncSetAttribute(dcn_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
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
    a.ctas = pl.ctas;
    a.total_units = pl.total_units;
    a.bn_total = pl.bn_total;
    a.nsub = pl.nsub;
    a.box_rows = pl.box_rows;
    a.stages = pl.stages;
    a.acc_cols = pl.acc_cols;
    a.tmem_cols = pl.tmem_cols;
    a.b_off = pl.b_off;
    a.info_off = pl.info_off;
    a.base_off = pl.base_off;
    a.bar_off = pl.bar_off;
    a.b_stage_bytes = pl.b_stage_bytes;
    dcn_fwd_tc_kernel<<<pl.ctas, NUM_THREADS, pl.smem_bytes, st>>>(map, a);
    if (launches) *launches += 2;
    return cudaGetLastError();
}

}  // namespace dcn
