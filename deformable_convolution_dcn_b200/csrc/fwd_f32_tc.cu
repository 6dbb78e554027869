// Forward DCNv2 in float32 on tcgen05 tensor cores for layers whose im2col
// depth K*K*Cin is at most 32 with Cin <= 3 (a 224x224 RGB stem layer is 27
// deep). The layer is Y[P x Cout] = Col[P x K*K*Cin] * W^T (the im2col view of
// the DCNv2 output equation); float32 accuracy comes from splitting both
// operands into a tf32 part and a float32 residual,
//
//   Col * W^T  ~=  Col_hi * W_hi^T + Col_hi * W_lo^T + Col_lo * W_hi^T,
//
// where x_hi is the nearest tf32 value of x and x_lo = x - x_hi (exact in
// float32). The dropped term Col_lo * W_lo^T and the tf32 reading of the
// residuals are each about 2^-21 of |Col||W|, far below the float32 tolerance.
//
// One CTA per 128 output pixels, 384 threads, three CTAs per SM:
//   * three threads share a tile row (pixel), each taking a third of the taps:
//     it loads those taps' offsets and mask, samples the bilinear neighbours
//     (all Cin channels, each neighbour outside the map contributing zero),
//     modulates them, and writes its values, split, into two 128-byte-swizzled
//     K-major A tiles;
//   * the CTA splits the weights [Cout, K*K*Cin] the same way into two B tiles;
//   * one thread issues the 12 tcgen05.mma (kind::tf32, M=128, N=Cout, K=8);
//   * each warp reads its 32 TMEM lanes back, adds the bias, and writes the rows
//     into a swizzled staging tile that two TMA tensor stores write to y (the
//     tile's rows are 128 consecutive output pixels, so y is written densely).
#include <cudaTypedefs.h>

#include <mutex>

#include "kernels.h"
#include "tc_ptx.cuh"

namespace dcn {
namespace {

constexpr int BM = 128;        // output pixels per CTA (UMMA M)
constexpr int KP = 32;         // padded contraction depth: one 128-byte swizzle row of float32
constexpr int PARTS = 3;       // threads per tile row, each gathering a third of the taps
constexpr int THREADS = PARTS * BM;
constexpr int TAPS_PER_PART = 3;  // ceil(MAX_TAPS / PARTS)
constexpr int MAX_TAPS = 9;
constexpr uint32_t TILE_BYTES = BM * 128;  // one [128 x 32] float32 swizzled tile
constexpr long long WAIT_LIMIT = 2000000000LL;

struct Args {
    Shape s;
    const float* x;
    const float* off;
    const float* mask;
    const float* w;
    const float* bias;
    unsigned* status;
    uint32_t b_off;      // B tiles after the A / staging region
    uint32_t w_off;      // raw weights [Cout][K*K*Cin] (bulk copy), after the B tiles
    uint32_t bar_off;
    int tmem_cols;
    int w_bulk;          // weights 16-byte aligned and a whole number of 16-byte units
};

// Byte offset of float32 element k of row r in a 128-byte-swizzled K-major tile:
// 16-byte chunk c of row r is stored at chunk c ^ (r % 8).
__device__ __forceinline__ uint32_t sw_chunk(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

template <int CIN>
__global__ void __launch_bounds__(THREADS, 3) stem_tc_kernel(const __grid_constant__ CUtensorMap tmap_y, const Args a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const Shape& s = a.s;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int KC = s.K2 * CIN;
    uint8_t* sA = smem;              // A_hi, A_lo (2 x 16 KB); afterwards the output staging tiles
    uint8_t* sB = smem + a.b_off;    // B_hi, B_lo (2 x Cout x 128 B)
    const uint32_t bsz = (uint32_t)s.Cout * 128;
    const float* sw = reinterpret_cast<const float*>(smem + a.w_off);
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + a.bar_off);   // MMA completion
    uint64_t* wbar = bar + 1;                                          // weights landed
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bar + 2);
    volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
    const uint32_t wbytes = (uint32_t)s.Cout * KC * 4;

    if (tid == 0) {
        ptx::mbar_init(ptx::smem_u32(bar), 1);
        ptx::mbar_init(ptx::smem_u32(wbar), 1);
        *s_abort = 0;
        ptx::fence_mbar_init();
        if (a.w_bulk) {
            // the weight matrix arrives while the offsets are loaded and the samples gathered
            ptx::mbar_arrive_expect_tx(ptx::smem_u32(wbar), wbytes);
            for (uint32_t o = 0; o < wbytes; o += 16384u)
                ptx::bulk_load(ptx::smem_u32(smem + a.w_off) + o, reinterpret_cast<const uint8_t*>(a.w) + o,
                               min(16384u, wbytes - o), ptx::smem_u32(wbar));
        }
    }
    if (warp == 0) {
        ptx::tmem_alloc(ptx::smem_u32(s_tmem), (uint32_t)a.tmem_cols);
        ptx::tmem_relinquish();
    }

    // ---- this thread's pixel and taps, their offsets and mask (all loads issued first)
    const int row = tid % BM, part = tid / BM;
    const int tp_lo = s.K2 * part / PARTS, tp_hi = s.K2 * (part + 1) / PARTS;
    const int plane = s.Ho * s.Wo;
    const int p = blockIdx.x * BM + row;
    const bool pv = p < s.P;
    int bb = 0, pix = 0, oy = 0, ox = 0;
    if (pv) {
        bb = p / plane;
        pix = p - bb * plane;
        const int ho = pix / s.Wo, wo = pix - ho * s.Wo;
        oy = ho * s.stride - s.pad;
        ox = wo * s.stride - s.pad;
    }
    const float* offp = a.off + (size_t)bb * 2 * s.K2 * plane + pix;
    const float* mp = a.mask ? a.mask + (size_t)bb * s.K2 * plane + pix : nullptr;
    float dy[TAPS_PER_PART], dx[TAPS_PER_PART], mk[TAPS_PER_PART];
#pragma unroll
    for (int j = 0; j < TAPS_PER_PART; ++j) {
        const int t = tp_lo + j;
        dy[j] = dx[j] = 0.f;
        mk[j] = 1.f;
        if (pv && t < tp_hi) {
            dy[j] = __ldg(offp + (size_t)(2 * t) * plane);
            dx[j] = __ldg(offp + (size_t)(2 * t + 1) * plane);
            if (mp) mk[j] = __ldg(mp + (size_t)t * plane);
        }
    }

    // ---- weights into B: row n = output channel, k = tap*Cin + c, zero for k >= KC
    __syncthreads();  // the weight barrier is initialised
    bool wok = true;
    if (a.w_bulk) wok = ptx::mbar_wait(ptx::smem_u32(wbar), 0, s_abort, a.status, WAIT_LIMIT);
    for (int e = tid; e < s.Cout * (KP / 4); e += THREADS) {
        const int n = e >> 3, c = e & 7;
        float v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int k = 4 * c + j;
            v[j] = k >= KC ? 0.f : (a.w_bulk ? sw[n * KC + k] : __ldg(a.w + (size_t)n * KC + k));
        }
        float hi[4], lo[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            hi[j] = ptx::to_tf32(v[j]);
            lo[j] = v[j] - hi[j];
        }
        const uint32_t o = ptx::smem_u32(sB) + sw_chunk(n, c);
        ptx::sts_v4(o, make_uint4(__float_as_uint(hi[0]), __float_as_uint(hi[1]), __float_as_uint(hi[2]),
                                  __float_as_uint(hi[3])));
        ptx::sts_v4(o + bsz, make_uint4(__float_as_uint(lo[0]), __float_as_uint(lo[1]), __float_as_uint(lo[2]),
                                        __float_as_uint(lo[3])));
    }

    // ---- this thread's modulated samples: k = tap*Cin + c for its taps
    const float* xb = a.x + (size_t)bb * s.H * s.W * CIN;
    const uint32_t arow = ptx::smem_u32(sA) + (uint32_t)row * 128;
#pragma unroll
    for (int j = 0; j < TAPS_PER_PART; ++j) {
        const int t = tp_lo + j;
        if (t >= tp_hi) break;
        float col[CIN];
#pragma unroll
        for (int c = 0; c < CIN; ++c) col[c] = 0.f;
        if (pv) {
            const int ti = t / s.K, tj = t - ti * s.K;
            int y0, x0;
            float ly, lx;
            split_coord(oy + ti * s.dil, dy[j], y0, ly);
            split_coord(ox + tj * s.dil, dx[j], x0, lx);
            float wt[4], v[4][CIN];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int r = y0 + (q >> 1), cc = x0 + (q & 1);
                wt[q] = 0.f;
#pragma unroll
                for (int c = 0; c < CIN; ++c) v[q][c] = 0.f;
                if (!inside(s, r, cc)) continue;
                wt[q] = ((q >> 1) ? ly : 1.f - ly) * ((q & 1) ? lx : 1.f - lx) * mk[j];
                const float* pc = xb + ((size_t)r * s.W + cc) * CIN;
#pragma unroll
                for (int c = 0; c < CIN; ++c) v[q][c] = __ldg(pc + c);
            }
#pragma unroll
            for (int c = 0; c < CIN; ++c)
                col[c] = wt[0] * v[0][c] + wt[1] * v[1][c] + wt[2] * v[2][c] + wt[3] * v[3][c];
        }
        // element k of the row: 16-byte chunk k/4 (swizzled by row), word k%4
#pragma unroll
        for (int c = 0; c < CIN; ++c) {
            const int k = t * CIN + c;
            const float hi = ptx::to_tf32(col[c]);
            const uint32_t o = arow + ((((k >> 2) ^ (row & 7)) << 4) | ((k & 3) << 2));
            ptx::sts_f32(o, hi);
            ptx::sts_f32(o + TILE_BYTES, col[c] - hi);
        }
    }
    if (part == PARTS - 1) {
        // zero padding of the contraction depth, in both A tiles
        for (int k = KC; k < KP; ++k) {
            const uint32_t o = arow + ((((k >> 2) ^ (row & 7)) << 4) | ((k & 3) << 2));
            ptx::sts_f32(o, 0.f);
            ptx::sts_f32(o + TILE_BYTES, 0.f);
        }
    }

    // ---- contraction on the tensor cores
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *s_tmem;
    if (tid == 0) {
        const uint32_t idesc = ptx::idesc_tf32_f32(BM, s.Cout);
        const uint32_t a0 = ptx::smem_u32(sA), b0 = ptx::smem_u32(sB);
        // small terms first; each K step of 8 tf32 is 32 bytes along the swizzled row
#pragma unroll
        for (int kk = 0; kk < KP / 8; ++kk)
            ptx::mma_tf32(tmem, ptx::sw128_desc(a0 + TILE_BYTES + kk * 32), ptx::sw128_desc(b0 + kk * 32), idesc,
                          kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < KP / 8; ++kk)
            ptx::mma_tf32(tmem, ptx::sw128_desc(a0 + kk * 32), ptx::sw128_desc(b0 + bsz + kk * 32), idesc, 1u);
#pragma unroll
        for (int kk = 0; kk < KP / 8; ++kk)
            ptx::mma_tf32(tmem, ptx::sw128_desc(a0 + kk * 32), ptx::sw128_desc(b0 + kk * 32), idesc, 1u);
        ptx::mma_commit(ptx::smem_u32(bar));
    }
    const bool ok = wok && ptx::mbar_wait(ptx::smem_u32(bar), 0, s_abort, a.status, WAIT_LIMIT);
    ptx::tc_fence_after();

    // ---- epilogue: TMEM -> registers (+ bias) -> swizzled staging -> TMA stores
    if (ok && warp < 4) {
        // warps 0-3 reach TMEM lanes 0-127 (a warp reads the lane quarter of its index mod 4)
        const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16);
        for (int cb = 0; cb < s.Cout / 32; ++cb) {
            float v[32];
            ptx::tmem_ld32(taddr + cb * 32, v);
            if (a.bias) {
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] += __ldg(a.bias + cb * 32 + j);
            }
            const uint32_t o = ptx::smem_u32(sA) + cb * TILE_BYTES;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                ptx::sts_v4(o + sw_chunk(tid, c), make_uint4(__float_as_uint(v[4 * c]), __float_as_uint(v[4 * c + 1]),
                                                             __float_as_uint(v[4 * c + 2]),
                                                             __float_as_uint(v[4 * c + 3])));
        }
        ptx::fence_proxy_async_smem();
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        if (ok) {
            for (int cb = 0; cb < s.Cout / 32; ++cb)
                ptx::tma_store_2d(&tmap_y, ptx::smem_u32(sA) + cb * TILE_BYTES, cb * 32, blockIdx.x * BM);
            ptx::bulk_commit_group();
            ptx::bulk_wait_group_read0();
        } else {
            // the MMAs were issued: let them finish (bounded) before TMEM is released
            volatile int dummy = 0;
            ptx::mbar_wait(ptx::smem_u32(bar), 0, &dummy, nullptr, WAIT_LIMIT);
        }
    }
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, (uint32_t)a.tmem_cols);
    }
}

struct Plan {
    uint32_t b_off, w_off, bar_off, smem_bytes;
    int tmem_cols;
};

Plan make_plan(const Shape& s) {
    Plan pl;
    const uint32_t stage = std::max<uint32_t>(2 * TILE_BYTES, (uint32_t)(s.Cout / 32) * TILE_BYTES);
    pl.b_off = stage;
    pl.w_off = pl.b_off + 2u * (uint32_t)s.Cout * 128;
    pl.bar_off = pl.w_off + (((uint32_t)s.Cout * s.K2 * s.Cin * 4 + 15) & ~15u);
    pl.smem_bytes = pl.bar_off + 64 + 1024;
    int cols = 32;
    while (cols < s.Cout) cols *= 2;
    pl.tmem_cols = cols;
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

template <int CIN>
cudaError_t launch(const Shape& s, const float* x, const float* off, const float* mask, const float* w,
                   const float* bias, float* y, unsigned* status, cudaStream_t st) {
    const Plan pl = make_plan(s);
    auto encode = get_encode();
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap map;
    cuuint64_t dims[2] = {(cuuint64_t)s.Cout, (cuuint64_t)s.P};
    cuuint64_t strides[1] = {(cuuint64_t)s.Cout * 4};
    cuuint32_t box[2] = {32, (cuuint32_t)BM};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, y, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    static DeviceFlags attr;
    cudaError_t e = max_dynamic_smem_once((const void*)stem_tc_kernel<CIN>, 227 * 1024, attr);
    if (e != cudaSuccess) return e;
    Args a;
    a.s = s;
    a.x = x;
    a.off = off;
    a.mask = mask;
    a.w = w;
    a.bias = bias;
    a.status = status;
    a.b_off = pl.b_off;
    a.w_off = pl.w_off;
    a.bar_off = pl.bar_off;
    a.w_bulk = ((reinterpret_cast<uintptr_t>(w) & 15) == 0 && ((size_t)s.Cout * s.K2 * s.Cin * 4) % 16 == 0) ? 1 : 0;
    a.tmem_cols = pl.tmem_cols;
    stem_tc_kernel<CIN><<<(s.P + BM - 1) / BM, THREADS, pl.smem_bytes, st>>>(map, a);
    return cudaGetLastError();
}

}  // namespace

// Cin <= 3 with one group, K*K <= 9, Cout a multiple of 32 up to 256, and
// index ranges within 32 bits (y must also be 16-byte aligned: TMA stores).
bool fwd_f32_tc_supported(const Shape& s) {
    if (s.Cin > 3 || s.G != 1 || s.K2 > MAX_TAPS || s.K2 * s.Cin > KP) return false;
    if (s.Cout % 32 || s.Cout < 32 || s.Cout > 256) return false;
    if ((long long)s.B * 2 * s.K2 * s.Ho * s.Wo >= (1LL << 31) || (long long)s.B * s.H * s.W * s.Cin >= (1LL << 31))
        return false;
    return make_plan(s).smem_bytes <= 227 * 1024;
}

cudaError_t fwd_f32_tc(const Shape& s, const void* x, const void* off, const void* mask, const void* w,
                       const void* bias, void* y, unsigned* status, cudaStream_t st) {
    // up to 128 output channels: the kernels of fwd_f32_stem.cu
    if (fwd_f32_stem_supported(s)) return fwd_f32_stem(s, x, off, mask, w, bias, y, status, st);
    const float *xf = (const float*)x, *of = (const float*)off, *mf = (const float*)mask, *wf = (const float*)w,
                *bf = (const float*)bias;
    float* yf = (float*)y;
    switch (s.Cin) {
        case 1: return launch<1>(s, xf, of, mf, wf, bf, yf, status, st);
        case 2: return launch<2>(s, xf, of, mf, wf, bf, yf, status, st);
        default: return launch<3>(s, xf, of, mf, wf, bf, yf, status, st);
    }
}

}  // namespace dcn
