// The offset/mask predictor of a bfloat16 DCNv2 layer with stride 1 as one
// tcgen05 kernel: the plain convolution with the layer's kernel size, padding
// and dilation and 3*G*K*K outputs (notes, DCNv2 section 3.2: the offsets and
// modulation scalars come from a separate convolution over the same input), with
// the sigmoid of the mask channels and the split into the offset and mask
// tensors fused into its epilogue.
//
// Implicit GEMM over the zero-padded input. Number the pixels of one padded
// image (Hp = H + 2 pad rows of Wp = W + 2 pad) in raster order; output pixel
// (ho, wo) then sits at padded index ho*Wp + wo, and tap (i, j) of it reads
// padded pixel ho*Wp + wo + i*dil*Wp + j*dil. A GEMM row m is a padded index, so
// for each tap the A operand of a 128-row tile is a window of 128 consecutive
// padded pixels, shifted by a constant: no im2col copy is made. Rows whose wo
// falls in the right-hand padding (wo >= Wo) are computed and discarded.
//
// One CTA per 128 GEMM rows of one image; per 64-channel slab of the input:
//   * one thread loads, by TMA, every padded row the tile's windows reach
//     (channels and rows outside the tensor read as zero: the padding) into a
//     128-byte-swizzled slab of 128-byte pixel rows, and the K*K weight tiles
//     [NP x 64 channels] (rows past 3GK^2 read as zero) into a ring;
//   * one thread issues, per tap, four tcgen05.mma (kind::f16, M=128, N=NP,
//     K=16) whose A descriptor starts at the tap's window inside the slab;
//   * four warps read the accumulator back from TMEM, add the bias and write
//     each valid pixel's offsets, and its masks through the sigmoid, in the
//     [B, C, Ho, Wo] layouts the layer reads.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "kernels.h"
#include "tc_ptx.cuh"

namespace dcn {
namespace {

constexpr int BM = 128;          // GEMM rows per CTA (UMMA M)
constexpr int THREADS = 192;     // warp 0: TMA, warp 1: MMA + TMEM, warps 2-5: epilogue
constexpr int XD = 2;            // input slab stages
constexpr int MAX_WD = 9;        // weight tile stages at most
constexpr long long WAIT_LIMIT = 2000000000LL;

struct PredArgs {
    Shape s;
    const bf16* bias;  // [nc] or null
    bf16* off;         // [B, no, Ho, Wo]
    bf16* mask;        // [B, nc - no, Ho, Wo]
    unsigned* status;
    int nc, no, np;    // outputs, offset outputs, UMMA N (nc rounded up to 16)
    int wp;            // padded width: the GEMM row pitch of one padded image row
    int nr;            // padded rows per input slab
    int tpi;           // tiles per image
    int ns;            // 64-channel slabs
    int wd;            // weight ring depth
    uint32_t xs_load;  // bytes of one input slab load (nr * wp * 128)
    uint32_t xs_bytes; // one input slab stage (1024-aligned)
    uint32_t wt_bytes; // one weight tile (np * 128)
    uint32_t w_off, bar_off;
    int tmem_cols;
};

// A window may start at any 128-byte row of a slab, inside a 1024-byte swizzle
// atom: the tensor cores take the swizzle phase of each row from its absolute
// shared-memory address bits (as TMA wrote it), so the plain descriptor, with
// the matrix base offset field left zero, reads the shifted window correctly
// (measured on B200: setting that field to the row's phase in the atom gives
// wrong sums).
__device__ __forceinline__ uint64_t window_desc(uint32_t saddr) { return ptx::sw128_desc(saddr); }

__global__ void __launch_bounds__(THREADS, 1)
    pred_tc_kernel(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmw, const PredArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const Shape& s = a.s;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + a.bar_off);
    const uint32_t xfull = ptx::smem_u32(bars), xempty = xfull + XD * 8;
    const uint32_t wfull = xempty + XD * 8, wempty = wfull + a.wd * 8;
    const uint32_t accb = wempty + a.wd * 8;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 2 * XD + 2 * a.wd + 1);
    volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
    const uint32_t xbase = ptx::smem_u32(smem), wbase = xbase + a.w_off;

    const int b = blockIdx.x / a.tpi;
    const int m0 = (blockIdx.x - b * a.tpi) * BM;  // first padded index of the tile in image b
    const int h0 = m0 / a.wp, r0 = m0 - h0 * a.wp;

    if (tid == 0) {
        for (int i = 0; i < 2 * XD + 2 * a.wd + 1; ++i) ptx::mbar_init(ptx::smem_u32(bars + i), 1);
        *s_abort = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&tmx);
        ptx::prefetch_tmap(&tmw);
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_u32(s_tmem), (uint32_t)a.tmem_cols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *s_tmem;

    if (warp == 0) {
        if (lane == 0) {
            // ---- TMA: per slab, the padded rows h0 .. h0+nr-1 (input rows shifted by -pad), then K*K weight tiles
            int xi = 0, wi = 0;
            bool ok = true;
            for (int sl = 0; sl < a.ns && ok; ++sl) {
                const int xs = xi % XD;
                if (xi >= XD) ok = ptx::mbar_wait(xempty + xs * 8, ((xi / XD) - 1) & 1, s_abort, a.status, WAIT_LIMIT);
                if (!ok) break;
                ptx::mbar_arrive_expect_tx(xfull + xs * 8, a.xs_load);
                ptx::tma_load_4d(xbase + xs * a.xs_bytes, &tmx, xfull + xs * 8, sl * 64, -s.pad, h0 - s.pad, b);
                ++xi;
                for (int t = 0; t < s.K2; ++t) {
                    const int ws = wi % a.wd;
                    if (wi >= a.wd)
                        ok = ptx::mbar_wait(wempty + ws * 8, ((wi / a.wd) - 1) & 1, s_abort, a.status, WAIT_LIMIT);
                    if (!ok) break;
                    ptx::mbar_arrive_expect_tx(wfull + ws * 8, a.wt_bytes);
                    ptx::tma_load_2d(wbase + ws * a.wt_bytes, &tmw, wfull + ws * 8, t * s.Cin + sl * 64, 0);
                    ++wi;
                }
            }
            // copies still in flight land before the CTA may exit (bounded)
            volatile int none = 0;
            for (int k = std::max(0, xi - XD); k < xi; ++k)
                ptx::mbar_wait(xfull + (k % XD) * 8, (k / XD) & 1, &none, nullptr, WAIT_LIMIT);
            for (int k = std::max(0, wi - a.wd); k < wi; ++k)
                ptx::mbar_wait(wfull + (k % a.wd) * 8, (k / a.wd) & 1, &none, nullptr, WAIT_LIMIT);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---- MMA: per slab and tap, A = the tap's 128-row window of the slab, B = the tap's weight tile
            const uint32_t idesc = ptx::idesc_bf16_f32(BM, a.np);
            int xi = 0, wi = 0;
            bool ok = true;
            for (int sl = 0; sl < a.ns && ok; ++sl) {
                const int xs = xi % XD;
                ok = ptx::mbar_wait(xfull + xs * 8, (xi / XD) & 1, s_abort, a.status, WAIT_LIMIT);
                if (!ok) break;
                ptx::tc_fence_after();
                const uint32_t slab = xbase + xs * a.xs_bytes;
                for (int t = 0; t < s.K2; ++t) {
                    const int ws = wi % a.wd;
                    ok = ptx::mbar_wait(wfull + ws * 8, (wi / a.wd) & 1, s_abort, a.status, WAIT_LIMIT);
                    if (!ok) break;
                    ptx::tc_fence_after();
                    const int i = t / s.K, j = t - i * s.K;
                    const uint32_t arow = slab + (uint32_t)(r0 + i * s.dil * a.wp + j * s.dil) * 128u;
                    const uint32_t wrow = wbase + ws * a.wt_bytes;
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        ptx::mma_bf16(tmem, window_desc(arow + k * 32), ptx::sw128_desc(wrow + k * 32), idesc,
                                      (sl | t | k) ? 1u : 0u);
                    ptx::mma_commit(wempty + ws * 8);
                    ++wi;
                }
                if (!ok) break;
                ptx::mma_commit(xempty + xs * 8);
                ++xi;
            }
            // always: arrives once every MMA issued above has completed
            ptx::mma_commit(accb);
        }
    } else {
        // ---- epilogue: warps 2-5 read TMEM lane quarters 2, 3, 0, 1 (a warp reaches quarter warp % 4)
        bool ok = ptx::mbar_wait(accb, 0, s_abort, a.status, WAIT_LIMIT);
        ptx::tc_fence_after();
        ok = __all_sync(0xffffffffu, ok && !*s_abort);
        if (ok) {
            const int q = warp & 3;
            const int pm = m0 + q * 32 + lane;
            const int ho = pm / a.wp, wo = pm - ho * a.wp;
            const bool valid = ho < s.Ho && wo < s.Wo;
            const int plane = s.Ho * s.Wo;
            const int nm = a.nc - a.no;
            bf16* offp = a.off + (size_t)b * a.no * plane + (valid ? ho * s.Wo + wo : 0);
            bf16* mp = a.mask + (size_t)b * nm * plane + (valid ? ho * s.Wo + wo : 0);
            const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16);
            for (int cb = 0; cb * 32 < a.nc; ++cb) {
                float v[32];
                ptx::tmem_ld32(taddr + cb * 32, v);
                if (valid) {
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        const int ch = cb * 32 + jj;
                        if (ch < a.nc) {
                            const float x = v[jj] + (a.bias ? __bfloat162float(a.bias[ch]) : 0.f);
                            if (ch < a.no)
                                offp[(size_t)ch * plane] = __float2bfloat16_rn(x);
                            else
                                mp[(size_t)(ch - a.no) * plane] = __float2bfloat16_rn(1.f / (1.f + expf(-x)));
                        }
                    }
                }
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        if (lane == 0) {
            // every issued MMA has completed before TMEM is released (bounded)
            volatile int none = 0;
            ptx::mbar_wait(accb, 0, &none, nullptr, WAIT_LIMIT);
        }
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, (uint32_t)a.tmem_cols);
    }
}

struct PredPlan {
    bool ok = false;
    int nc, no, np, wp, nr, tpi, ns, wd, tmem_cols;
    uint32_t xs_load, xs_bytes, wt_bytes, w_off, bar_off, smem;
    long long grid;
};

PredPlan make_pred_plan(const Shape& s) {
    PredPlan p;
    if (s.stride != 1 || s.Cin % 8 || s.K2 > 64) return p;
    p.nc = 3 * s.G * s.K2;
    p.no = 2 * s.G * s.K2;
    p.np = (p.nc + 15) / 16 * 16;
    if (p.np > 256) return p;
    p.wp = s.W + 2 * s.pad;
    if (p.wp > 256 || s.Wo != p.wp - s.dil * (s.K - 1)) return p;
    // the windows of a tile reach padded indices r0 .. r0 + 127 + dil*(K-1)*(Wp+1), r0 < Wp
    const long long reach = (long long)p.wp - 1 + BM + (long long)s.dil * (s.K - 1) * (p.wp + 1);
    p.nr = (int)((reach + p.wp - 1) / p.wp);
    if (p.nr > 256) return p;
    p.xs_load = (uint32_t)p.nr * p.wp * 128u;
    p.xs_bytes = (p.xs_load + 1023u) & ~1023u;
    p.wt_bytes = (uint32_t)p.np * 128u;
    p.ns = (s.Cin + 63) / 64;
    const uint32_t xtot = XD * p.xs_bytes;
    // two CTAs per SM when the ring still holds four weight tiles in half the shared memory
    const uint32_t half = 110u * 1024u, full = 220u * 1024u;
    const uint32_t lim = (xtot + 4u * p.wt_bytes <= half) ? half : full;
    if (xtot + 2u * p.wt_bytes > lim) return p;
    p.wd = (int)std::min<uint32_t>(MAX_WD, (lim - xtot) / p.wt_bytes);
    p.wd = std::min(p.wd, s.K2 * p.ns);
    p.wd = std::max(p.wd, 2);
    p.w_off = xtot;
    p.bar_off = p.w_off + (uint32_t)p.wd * p.wt_bytes;
    p.smem = p.bar_off + (uint32_t)(2 * XD + 2 * p.wd + 1) * 8u + 16u + 1024u;
    int cols = 32;
    while (cols < p.np) cols *= 2;
    p.tmem_cols = cols;
    p.tpi = (int)(((long long)s.Ho * p.wp + BM - 1) / BM);
    p.grid = (long long)s.B * p.tpi;
    if (p.grid >= (1LL << 31) || (long long)s.Ho * p.wp + BM >= (1LL << 31)) return p;
    p.ok = p.smem <= 227u * 1024u;
    return p;
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

}  // namespace

bool pred_tc_supported(const Shape& s) { return make_pred_plan(s).ok; }

cudaError_t pred_tc(const Shape& s, const void* x, const void* w, const void* bias, void* off, void* mask,
                    unsigned* status, cudaStream_t st) {
    const PredPlan pl = make_pred_plan(s);
    if (!pl.ok) return cudaErrorInvalidValue;
    auto encode = encode_fn();
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap mx, mw;
    {
        cuuint64_t dims[4] = {(cuuint64_t)s.Cin, (cuuint64_t)s.W, (cuuint64_t)s.H, (cuuint64_t)s.B};
        cuuint64_t strides[3] = {(cuuint64_t)s.Cin * 2, (cuuint64_t)s.W * s.Cin * 2, (cuuint64_t)s.H * s.W * s.Cin * 2};
        cuuint32_t box[4] = {64, (cuuint32_t)pl.wp, (cuuint32_t)pl.nr, 1};
        cuuint32_t estr[4] = {1, 1, 1, 1};
        if (encode(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(x), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        cuuint64_t dims[2] = {(cuuint64_t)s.KC, (cuuint64_t)pl.nc};
        cuuint64_t strides[1] = {(cuuint64_t)s.KC * 2};
        cuuint32_t box[2] = {64, (cuuint32_t)pl.np};
        cuuint32_t estr[2] = {1, 1};
        if (encode(&mw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(w), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    static DeviceFlags attr;
    cudaError_t e = max_dynamic_smem_once((const void*)pred_tc_kernel, 227 * 1024, attr);
    if (e != cudaSuccess) return e;
    PredArgs a;
    a.s = s;
    a.bias = (const bf16*)bias;
    a.off = (bf16*)off;
    a.mask = (bf16*)mask;
    a.status = status;
    a.nc = pl.nc;
    a.no = pl.no;
    a.np = pl.np;
    a.wp = pl.wp;
    a.nr = pl.nr;
    a.tpi = pl.tpi;
    a.ns = pl.ns;
    a.wd = pl.wd;
    a.xs_load = pl.xs_load;
    a.xs_bytes = pl.xs_bytes;
    a.wt_bytes = pl.wt_bytes;
    a.w_off = pl.w_off;
    a.bar_off = pl.bar_off;
    a.tmem_cols = pl.tmem_cols;
    pred_tc_kernel<<<(unsigned)pl.grid, THREADS, pl.smem, st>>>(mx, mw, a);
    return cudaGetLastError();
}

}  // namespace dcn
