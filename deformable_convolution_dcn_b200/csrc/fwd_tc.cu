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

constexpr int BM = 128;                 // output pixels per tile (UMMA M); row index = e & 127 below
constexpr int BK = 64;                  // bf16 per K chunk (one 128-byte swizzle row)
constexpr int A_STAGE_BYTES = BM * BK * 2;
constexpr int NUM_PROD_WARPS = 8;
constexpr int TMA_WARP = 4, MMA_WARP = 5, PROD_WARP0 = 6;  // warps 0-3: epilogue
constexpr int NUM_THREADS = (PROD_WARP0 + NUM_PROD_WARPS) * 32;
constexpr int NUM_PROD_THREADS = NUM_PROD_WARPS * 32;
#ifndef DCN_FWD_GROUPS
#define DCN_FWD_GROUPS 2
#endif
#ifndef DCN_FWD_BLEND
#define DCN_FWD_BLEND 1
#endif
constexpr int GROUPS = DCN_FWD_GROUPS;                    // producer groups taking alternate chunks
constexpr int GROUP_THREADS = NUM_PROD_THREADS / GROUPS;
constexpr int ROW_STEP = GROUP_THREADS / 8;                 // rows between a thread's rows
constexpr int ROWS_PER_THREAD = BM / ROW_STEP;
constexpr int INFO_BATCH = 5;
#ifndef DCN_FWD_PREFETCH
#define DCN_FWD_PREFETCH 1
#endif
constexpr bool PREFETCH = DCN_FWD_PREFETCH != 0;           // L1 prefetch of the next chunk's neighbours                               // sampling records per thread per pass
constexpr long long WAIT_LIMIT = 2000000000LL;  // clock cycles (about a second)
constexpr int MAX_STAGES = 8;
#ifndef DCN_FWD_MAX_STAGES
#define DCN_FWD_MAX_STAGES 3
#endif

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
    int sw, nf, wl;    // pixel order: vertical strips of width sw (nf full strips, last one wl wide)
    long long total_units;
    int bn_total;      // tile width in output channels (multiple of 16, <= 512)
    int nsub;          // accumulators per tile (1: N = bn_total; 2: 256 + rest)
    int box_rows;      // rows of one weight box
    int stages;
    int acc_cols;      // TMEM column stride between the two accumulator buffers (0: single buffer)
    int tmem_cols;
    uint32_t b_off, info_off, base_off, row_off, bar_off, b_stage_bytes;
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

// Modulated bilinear blend of one row's four neighbour vectors (8 channels
// each) into 8 bf16 values. DCN_FWD_BLEND == 1: packed bf16x2 FMAs (each
// partial sum rounded to bf16); 0: bf16 products accumulated in f32.
__device__ __forceinline__ uint4 blend4(const uint4 (&v)[4], const TapW& tw) {
#if DCN_FWD_BLEND
    const uint32_t w00 = __byte_perm(tw.w01_00, 0, 0x1010), w01 = __byte_perm(tw.w01_00, 0, 0x3232);
    const uint32_t w10 = __byte_perm(tw.w11_10, 0, 0x1010), w11 = __byte_perm(tw.w11_10, 0, 0x3232);
    const uint32_t* a0 = reinterpret_cast<const uint32_t*>(&v[0]);
    const uint32_t* a1 = reinterpret_cast<const uint32_t*>(&v[1]);
    const uint32_t* a2 = reinterpret_cast<const uint32_t*>(&v[2]);
    const uint32_t* a3 = reinterpret_cast<const uint32_t*>(&v[3]);
    uint32_t r[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        asm("{\n\t"
            "mul.rn.bf16x2 %0, %1, %5;\n\t"
            "fma.rn.bf16x2 %0, %2, %6, %0;\n\t"
            "fma.rn.bf16x2 %0, %3, %7, %0;\n\t"
            "fma.rn.bf16x2 %0, %4, %8, %0;\n\t}"
            : "=&r"(r[q])
            : "r"(a0[q]), "r"(a1[q]), "r"(a2[q]), "r"(a3[q]), "r"(w00), "r"(w01), "r"(w10), "r"(w11));
    }
    return make_uint4(r[0], r[1], r[2], r[3]);
#else
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    fma8(acc, v[0], tw.w01_00, false);
    fma8(acc, v[1], tw.w01_00, true);
    fma8(acc, v[2], tw.w11_10, false);
    fma8(acc, v[3], tw.w11_10, true);
    return make_uint4(pack_bf16(acc[0], acc[1]), pack_bf16(acc[2], acc[3]), pack_bf16(acc[4], acc[5]),
                      pack_bf16(acc[6], acc[7]));
#endif
}

// GEMM rows enumerate output pixels strip by strip: each image is cut into
// vertical strips sw pixels wide, rows of a strip are consecutive, so a tile of
// 128 rows covers a compact block of pixels whose bilinear neighbourhoods
// overlap in L1. Returns the raster index (b*Ho + ho)*Wo + wo, or -1 past the end.
__device__ __forceinline__ int strip_to_raster(int idx, const FwdArgs& a) {
    const Shape& s = a.s;
    if (idx >= s.P) return -1;
    const int plane = s.Ho * s.Wo;
    const int b = idx / plane;
    const int rem = idx - b * plane;
    const int full = a.nf * s.Ho * a.sw;
    int ho, wo;
    if (rem < full) {
        const int strip = rem / (s.Ho * a.sw);
        const int r2 = rem - strip * (s.Ho * a.sw);
        ho = r2 / a.sw;
        wo = strip * a.sw + (r2 - ho * a.sw);
    } else {
        const int r2 = rem - full;
        ho = r2 / a.wl;
        wo = a.nf * a.sw + (r2 - ho * a.wl);
    }
    return (b * s.Ho + ho) * s.Wo + wo;
}

// Partial tiles (float32) live in the workspace as [cta][slot][bn_total/32][8][BM][4]:
// slot 0 holds a CTA's first segment, slot 1 its last; within a tile, the four
// consecutive columns 4q..4q+3 of a 32-column block are stored for all 128
// rows side by side, so each warp-wide 16-byte access covers 512 contiguous bytes.
__device__ __forceinline__ const float* partial_base(const FwdArgs& a, int c, long long tu0, int row) {
    const int slot = (unit_begin(c, a) >= tu0) ? 0 : 1;
    return a.partials + ((size_t)c * 2 + slot) * BM * a.bn_total + (size_t)row * 4;
}

// v[0..31] += partial columns cc..cc+31 of this row (src from partial_base).
__device__ __forceinline__ void add_partial32(float (&v)[32], const float* src, int cc) {
    float4 f[8];
    const float* b = src + (size_t)(cc >> 5) * 8 * BM * 4;
#pragma unroll
    for (int q = 0; q < 8; ++q) f[q] = ptx::ldcg_f4(b + q * BM * 4);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        v[4 * q] += f[q].x;
        v[4 * q + 1] += f[q].y;
        v[4 * q + 2] += f[q].z;
        v[4 * q + 3] += f[q].w;
    }
}

// As add_partial32, from a partial tile staged in shared memory.
__device__ __forceinline__ void add_partial32_smem(float (&v)[32], const float* src, int cc) {
    const float* b = src + (size_t)(cc >> 5) * 8 * BM * 4;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const float4 f = *reinterpret_cast<const float4*>(b + q * BM * 4);
        v[4 * q] += f.x;
        v[4 * q + 1] += f.y;
        v[4 * q + 2] += f.z;
        v[4 * q + 3] += f.w;
    }
}

// y[row, n0 + cc .. n0 + cc + 31] = v + bias, as bf16 (columns < ncols).
__device__ __forceinline__ void store_row32(bf16* yrow, int cc, int ncols, float (&v)[32], const bf16* bias, int n0) {
    if (bias) {
#pragma unroll
        for (int e = 0; e < 32; ++e)
            if (cc + e < ncols) v[e] += __bfloat162float(bias[n0 + cc + e]);
    }
    if (cc + 32 <= ncols) {
        uint4* dst = reinterpret_cast<uint4*>(yrow + cc);
#pragma unroll
        for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(pack_bf16(v[8 * q], v[8 * q + 1]), pack_bf16(v[8 * q + 2], v[8 * q + 3]),
                                pack_bf16(v[8 * q + 4], v[8 * q + 5]), pack_bf16(v[8 * q + 6], v[8 * q + 7]));
    } else {
#pragma unroll
        for (int e = 0; e < 32; ++e)
            if (cc + e < ncols) yrow[cc + e] = __float2bfloat16_rn(v[e]);
    }
}

// Barrier among the four epilogue warps (an mbarrier with a bounded wait).
__device__ __forceinline__ bool epi_sync(uint64_t* bar, uint32_t& ph, volatile int* abort, unsigned* status) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) ptx::mbar_arrive(ptx::smem_u32(bar));
    const bool ok = ptx::mbar_wait(ptx::smem_u32(bar), ph, abort, status, WAIT_LIMIT);
    ph ^= 1;
    return ok;
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
    int4* s_row = reinterpret_cast<int4*>(smem + a.row_off);   // per tile row: in-plane pixel, b, row/col origin
    int2* s_tap = reinterpret_cast<int2*>(s_row + BM);          // per tap: (i*dil, j*dil)
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + a.bar_off);
    // barrier slots
    uint64_t* full_a = bars;
    uint64_t* tail_bar = bars + MAX_STAGES;  // bulk copy of other CTAs' partials for the last segment
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
            // a stage is full when its producer group's warps and the weight TMA have both arrived
            ptx::mbar_init(ptx::smem_u32(&full_a[i]), NUM_PROD_WARPS / GROUPS + 1);
            ptx::mbar_init(ptx::smem_u32(&empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(ptx::smem_u32(&acc_full[i]), 1);
            ptx::mbar_init(ptx::smem_u32(&acc_empty[i]), 4);
        }
        ptx::mbar_init(ptx::smem_u32(drain), 1);
        ptx::mbar_init(ptx::smem_u32(tail_bar), 1);
        ptx::mbar_init(ptx::smem_u32(prod_bar), NUM_PROD_WARPS);
        ptx::mbar_init(ptx::smem_u32(epi_bar), 4);
        *s_abort = 0;
        *s_last = 0;
        ptx::fence_mbar_init();
    }
    if (threadIdx.x < s.K2) {
        const int i = threadIdx.x / s.K;
        s_tap[threadIdx.x] = make_int2(i * s.dil, (threadIdx.x - i * s.K) * s.dil);
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
        // Two groups of producer warps take alternate chunks, so that one group
        // blends while the other's loads are in flight. Within a group, 8 lanes
        // cover the 128-byte channel slice of one row (one 16-byte vector each).
        const int ptid = threadIdx.x - PROD_WARP0 * 32;
        const int plane = s.Ho * s.Wo;
        const int grp = ptid / GROUP_THREADS;
        const int gtid = ptid - grp * GROUP_THREADS;
        const int j = gtid & 7, r0 = gtid >> 3;
        int stage = 0;
        uint32_t phase = 0, pphase = 0;
        int n = 0;  // chunk sequence number within this CTA
        bool ok = true;
        for (long long u = ubeg; u < uend && ok;) {
            const int t = (int)(u / a.U);
            const int k0 = (int)(u - (long long)t * a.U);
            const int k1 = (int)min((long long)a.U, uend - (long long)t * a.U);
            const int mt = t / a.n_tiles;
            int cur_g = -1;
            Chunk ch = chunk_of(k0, a);
            for (int k = k0; k < k1 && ok; ++k) {
                if (ch.g != cur_g) {
                    // every producer is done with the previous records before they are overwritten
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(prod_bar));
                    if (!ptx::mbar_wait(ptx::smem_u32(prod_bar), pphase, s_abort, a.status, WAIT_LIMIT)) {
                        ok = false;
                        break;
                    }
                    pphase ^= 1;
                    if (cur_g < 0) {
                        // new tile: pixel coordinates of its rows
                        if (ptid < BM) {
                            const int pr = strip_to_raster(mt * BM + ptid, a);
                            int4 ri = make_int4(-1, 0, 0, 0);
                            if (pr >= 0) {
                                const int bb = pr / plane, pix = pr - bb * plane;
                                const int ho = pix / s.Wo, wo = pix - ho * s.Wo;
                                ri = make_int4(pix, bb, ho * s.stride - s.pad, wo * s.stride - s.pad);
                            }
                            s_row[ptid] = ri;
                        }
                        __syncwarp();
                        if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(prod_bar));
                        if (!ptx::mbar_wait(ptx::smem_u32(prod_bar), pphase, s_abort, a.status, WAIT_LIMIT)) {
                            ok = false;
                            break;
                        }
                        pphase ^= 1;
                    }
                    // sampling records of every (row, tap) of this tile for group ch.g; each
                    // thread issues the loads of all its entries before using any of them
                    for (int e0 = 0; e0 < BM * s.K2; e0 += INFO_BATCH * NUM_PROD_THREADS) {
                        float dy[INFO_BATCH], dx[INFO_BATCH], mk[INFO_BATCH];
#pragma unroll
                        for (int b = 0; b < INFO_BATCH; ++b) {
                            const int e = e0 + b * NUM_PROD_THREADS + ptid;
                            const int tp = e >> 7, row = e & (BM - 1);
                            dy[b] = dx[b] = 0.f;
                            mk[b] = 1.f;
                            if (e < BM * s.K2) {
                                const int4 ri = s_row[row];
                                if (ri.x >= 0) {
                                    const size_t ob =
                                        ((size_t)ri.y * 2 * s.G * s.K2 + (size_t)ch.g * 2 * s.K2 + 2 * tp) * plane + ri.x;
                                    dy[b] = __bfloat162float(a.off[ob]);
                                    dx[b] = __bfloat162float(a.off[ob + plane]);
                                    if (a.mask)
                                        mk[b] = __bfloat162float(
                                            a.mask[((size_t)ri.y * s.G * s.K2 + (size_t)ch.g * s.K2 + tp) * plane + ri.x]);
                                }
                            }
                        }
#pragma unroll
                        for (int b = 0; b < INFO_BATCH; ++b) {
                            const int e = e0 + b * NUM_PROD_THREADS + ptid;
                            if (e >= BM * s.K2) continue;
                            const int tp = e >> 7, row = e & (BM - 1);
                            const int4 ri = s_row[row];
                            float w00 = 0.f, w01 = 0.f, w10 = 0.f, w11 = 0.f;
                            int base = 0;
                            if (ri.x >= 0) {
                                const int2 to = s_tap[tp];
                                int y0, x0;
                                float ly, lx;
                                split_coord(ri.z + to.x, dy[b], y0, ly);
                                split_coord(ri.w + to.y, dx[b], x0, lx);
                                const bool v00 = inside(s, y0, x0), v01 = inside(s, y0, x0 + 1);
                                const bool v10 = inside(s, y0 + 1, x0), v11 = inside(s, y0 + 1, x0 + 1);
                                w00 = v00 ? (1.f - ly) * (1.f - lx) * mk[b] : 0.f;
                                w01 = v01 ? (1.f - ly) * lx * mk[b] : 0.f;
                                w10 = v10 ? ly * (1.f - lx) * mk[b] : 0.f;
                                w11 = v11 ? ly * lx * mk[b] : 0.f;
                                if (v00 | v01 | v10 | v11) base = (ri.y * s.H + y0) * s.W + x0;
                            }
                            TapW tw;
                            tw.w01_00 = pack_bf16(w00, w01);
                            tw.w11_10 = pack_bf16(w10, w11);
                            s_w[row * s.K2 + tp] = tw;
                            s_base[row * s.K2 + tp] = base;
                        }
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
                if ((n % GROUPS) == grp) {
                    if (!ptx::mbar_wait(ptx::smem_u32(&empty[stage]), phase ^ 1, s_abort, a.status, WAIT_LIMIT)) {
                        ok = false;
                        break;
                    }
                    const int cg = ch.q * BK + j * 8;  // channel within the group
                    const bool cval = cg < s.Cg;
                    const bf16* xc = a.x + ch.g * s.Cg + cg;
                    const long long rowpitch = (long long)s.W * s.Cin;
                    const uint32_t a_stage = ptx::smem_u32(sA + stage * A_STAGE_BYTES);
#pragma unroll
                    for (int bt = 0; bt < ROWS_PER_THREAD / 4; ++bt) {
                        uint4 v[4][4];
                        TapW tw[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int row = r0 + ROW_STEP * (4 * bt + i);
                            tw[i] = s_w[row * s.K2 + ch.tap];
                            const int base = s_base[row * s.K2 + ch.tap];
                            const bf16* pb = xc + (long long)base * s.Cin;
                            uint32_t m = ((tw[i].w01_00 & 0xFFFFu) ? 1u : 0u) | ((tw[i].w01_00 >> 16) ? 2u : 0u) |
                                         ((tw[i].w11_10 & 0xFFFFu) ? 4u : 0u) | ((tw[i].w11_10 >> 16) ? 8u : 0u);
                            if (!cval) m = 0;
                            ptx::ldg4_pred(v[i], pb, pb + s.Cin, pb + rowpitch, pb + rowpitch + s.Cin, m);
                        }
                        if (bt == 0 && PREFETCH) {
                            // Pull the neighbours of this group's next chunk into L1 while this one
                            // is blended: lane j takes row r0 + ROW_STEP*j, all four corners.
                            Chunk nx = ch;
                            int kn = k;
                            for (int d = 0; d < GROUPS; ++d) {
                                ++kn;
                                if (++nx.tap == s.K2) {
                                    nx.tap = 0;
                                    if (++nx.q == a.nq) {
                                        nx.q = 0;
                                        ++nx.g;
                                    }
                                }
                            }
                            const int cgn = nx.q * BK;
                            if (kn < k1 && nx.g == ch.g && cgn < s.Cg && j < ROWS_PER_THREAD) {
                                const int row = r0 + ROW_STEP * j;
                                const TapW tn = s_w[row * s.K2 + nx.tap];
                                const bf16* pn = a.x + (long long)s_base[row * s.K2 + nx.tap] * s.Cin + ch.g * s.Cg + cgn;
                                if (tn.w01_00 & 0xFFFFu) ptx::prefetch_l1(pn);
                                if (tn.w01_00 >> 16) ptx::prefetch_l1(pn + s.Cin);
                                if (tn.w11_10 & 0xFFFFu) ptx::prefetch_l1(pn + rowpitch);
                                if (tn.w11_10 >> 16) ptx::prefetch_l1(pn + rowpitch + s.Cin);
                            }
                        }
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int row = r0 + ROW_STEP * (4 * bt + i);
                            ptx::sts_v4(a_stage + row * 128 + ((j ^ (row & 7)) << 4), blend4(v[i], tw[i]));
                        }
                    }
                    ptx::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&full_a[stage]));
                }
                if (++stage == a.stages) {
                    stage = 0;
                    phase ^= 1;
                }
                ++n;
                if (++ch.tap == s.K2) {
                    ch.tap = 0;
                    if (++ch.q == a.nq) {
                        ch.q = 0;
                        ++ch.g;
                    }
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
                u = (long long)t * a.U + k1;
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
                    if (!ptx::mbar_wait(ptx::smem_u32(&full_a[stage]), phase, s_abort, a.status, WAIT_LIMIT)) {
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
            const int p = strip_to_raster(mt * BM + row, a);
            const uint32_t taddr = tmem_base + (uint32_t)(abuf * a.acc_cols) + ((uint32_t)(quarter * 32) << 16);
            const bool full = (k0 == 0 && k1 == a.U);
            const int ncols = min(a.bn_total, s.Cout - n0);
            bf16* yrow = a.y + (size_t)(p < 0 ? 0 : p) * s.Cout + n0;
            if (full) {
                for (int cc = 0; cc < a.bn_total; cc += 32) {
                    float v[32];
                    ptx::tmem_ld32(taddr + cc, v);
                    if (p >= 0 && cc < ncols) store_row32(yrow, cc, ncols, v, a.bias, n0);
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&acc_empty[abuf]));
            } else {
                const long long tu0 = (long long)t * a.U;
                const int c_lo = cta_of_unit(tu0, a), c_hi = cta_of_unit(tu0 + a.U - 1, a);
                // If every other contributor of this tile has already published its
                // partial, add them to this CTA's accumulator straight from TMEM.
                if (threadIdx.x == 0) *s_last = (ptx::ld_acquire_gpu(a.counters + t) == c_hi - c_lo) ? 1 : 0;
                if (!epi_sync(epi_bar, ephase, s_abort, a.status)) {
                    ok = false;
                    break;
                }
                if (*s_last) {
                    // The CTA's last segment: the pipeline buffers are idle, so when the other
                    // contributors' partial tiles fit there they are bulk-copied in and read
                    // from shared memory; otherwise they are read from global memory.
                    const uint32_t tile_bytes = (uint32_t)BM * a.bn_total * 4;
                    const bool last_seg = (long long)t * a.U + k1 == uend;
                    const bool staged = last_seg && (uint32_t)(c_hi - c_lo) * tile_bytes <= a.b_off + a.stages * a.b_stage_bytes;
                    if (staged) {
                        if (threadIdx.x == 0) {
                            ptx::fence_proxy_async_all();
                            const uint32_t tb = ptx::smem_u32(tail_bar);
                            ptx::mbar_arrive_expect_tx(tb, (uint32_t)(c_hi - c_lo) * tile_bytes);
                            uint32_t dst = ptx::smem_u32(smem);
                            for (int c = c_lo; c <= c_hi; ++c) {
                                if (c == cta) continue;
                                const uint8_t* src = reinterpret_cast<const uint8_t*>(partial_base(a, c, tu0, 0));
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
                    for (int cc = 0; cc < ncols; cc += 32) {
                        float v[32];
                        ptx::tmem_ld32(taddr + cc, v);
                        int slot = 0;
                        for (int c = c_lo; c <= c_hi; ++c) {
                            if (c == cta) continue;
                            if (staged)
                                add_partial32_smem(v, reinterpret_cast<const float*>(smem + (size_t)slot * tile_bytes) + row * 4, cc);
                            else
                                add_partial32(v, partial_base(a, c, tu0, row), cc);
                            ++slot;
                        }
                        if (p >= 0) store_row32(yrow, cc, ncols, v, a.bias, n0);
                    }
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&acc_empty[abuf]));
                    if (threadIdx.x == 0) a.counters[t] = 0;
                } else {
                    float* dst = const_cast<float*>(partial_base(a, cta, tu0, row));
                    for (int cc = 0; cc < a.bn_total; cc += 32) {
                        float v[32];
                        ptx::tmem_ld32(taddr + cc, v);
                        float* b = dst + (size_t)(cc >> 5) * 8 * BM * 4;
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            *reinterpret_cast<float4*>(b + q * BM * 4) =
                                make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                    }
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&acc_empty[abuf]));
                    __threadfence();
                    if (!epi_sync(epi_bar, ephase, s_abort, a.status)) {
                        ok = false;
                        break;
                    }
                    if (threadIdx.x == 0) *s_last = (atomicAdd(a.counters + t, 1) == c_hi - c_lo) ? 1 : 0;
                    if (!epi_sync(epi_bar, ephase, s_abort, a.status)) {
                        ok = false;
                        break;
                    }
                    if (*s_last) {
                        __threadfence();
                        if (p >= 0) {
                            for (int cc = 0; cc < ncols; cc += 32) {
                                float v[32];
#pragma unroll
                                for (int e = 0; e < 32; ++e) v[e] = 0.f;
                                for (int c = c_lo; c <= c_hi; ++c) add_partial32(v, partial_base(a, c, tu0, row), cc);
                                store_row32(yrow, cc, ncols, v, a.bias, n0);
                            }
                        }
                        if (threadIdx.x == 0) a.counters[t] = 0;
                    }
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
    int sw, nf, wl;
    long long total_units;
    uint32_t b_off, info_off, base_off, row_off, bar_off, b_stage_bytes, smem_bytes;
    size_t ws_partials, ws_counters_off, ws_bytes;
};

Plan make_plan(const Shape& s, int sms) {
    Plan pl{};
    pl.ok = false;
    if (s.Cin % 8 || s.Cg % 8 || s.Cout % 8 || s.K2 > 25) return pl;
    pl.bn_total = std::min(512, (s.Cout + 31) / 32 * 32);
    pl.n_tiles = (s.Cout + pl.bn_total - 1) / pl.bn_total;
    pl.m_tiles = (s.P + BM - 1) / BM;
    pl.tiles = pl.m_tiles * pl.n_tiles;
    pl.nq = (s.Cg + BK - 1) / BK;
    // strip width: a divisor of Wo in [8, 16] if there is one, else 12 (or Wo when narrower)
    pl.sw = std::min(s.Wo, 12);
    if (s.Wo > 16) {
        for (int c = 8; c <= 16; ++c)
            if (s.Wo % c == 0) pl.sw = c;
    }
    pl.nf = s.Wo / pl.sw;
    pl.wl = s.Wo - pl.nf * pl.sw;
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
    const uint32_t fixed = info_bytes + BM * 16 + 256 + 64 * 8 + 64 + 1024;  // info, barriers, flags, alignment slack
    const uint32_t budget = 227 * 1024;
    const uint32_t stage_bytes = A_STAGE_BYTES + pl.b_stage_bytes;
    int st = (int)((budget - fixed) / stage_bytes);
    st = std::min(st, DCN_FWD_MAX_STAGES);
    if (st < 2) return pl;
    pl.stages = st;
    pl.b_off = (uint32_t)(st * A_STAGE_BYTES);
    pl.info_off = pl.b_off + (uint32_t)st * pl.b_stage_bytes;
    pl.base_off = pl.info_off + (uint32_t)(BM * s.K2 * sizeof(TapW));
    pl.row_off = (pl.base_off + (uint32_t)(BM * s.K2 * sizeof(int)) + 15) & ~15u;
    pl.bar_off = (pl.row_off + (uint32_t)(BM * sizeof(int4) + 32 * sizeof(int2)) + 7) & ~7u;
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
    a.sw = pl.sw;
    a.nf = pl.nf;
    a.wl = pl.wl;
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
    a.row_off = pl.row_off;
    a.bar_off = pl.bar_off;
    a.b_stage_bytes = pl.b_stage_bytes;
    dcn_fwd_tc_kernel<<<pl.ctas, NUM_THREADS, pl.smem_bytes, st>>>(map, a);
    if (launches) *launches += 2;
    return cudaGetLastError();
}


// ------------------------------------------------- forward without allocation --
// Scratch for callers that cannot allocate device memory themselves (see
// dcn_forward_noalloc in include/dcn.h). The array lives in this module's
// device image, so every GPU that loads the library holds it until the
// process exits; all calls share it.
namespace {

constexpr size_t kStaticScratchBytes = 40ull << 20;  // 40 MiB
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
