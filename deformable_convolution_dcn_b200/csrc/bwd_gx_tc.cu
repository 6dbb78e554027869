// grad_x of DCNv2 on sm_100a tensor cores (bfloat16 in, float32 out), with the
// bilinear scatter accumulated in shared memory.
//
// grad_x[b, r, c, ch] = sum over the samples (p, tap) whose bilinear footprint
// holds (r, c) of G[p, tap, ch] * m * w_corner, with the column gradient
// G = grad_y * W (the col2im side of the im2col view in the "Deformable
// ConvNets" notes; the four neighbours of a sample carry its gradient, a
// neighbour outside the map none). Adding every (pixel, tap, channel, corner)
// term into grad_x with a global atomic costs one L2 atomic per 16 bytes
// (about 46 M for the ResNet-50 conv4 layer); here the terms of one work unit
// are first summed in a float32 window of grad_x held in shared memory, which
// is added to grad_x once, with 16-byte vector atomics, when the unit ends.
//
// Unit = (128 output pixels in raster order, 32 input channels of one group).
// Its window covers the input rows the unit's samples can reach (the rows of
// its output pixels, widened by the kernel's reach and a margin for the
// offsets), full width, capped at WIN_CELLS pixels; a corner outside the
// window (an offset beyond the margin, a pixel of another image) goes to
// grad_x directly with a scalar atomic.
//
//   * TMA warp: grad_y tiles [128 x 64] (A, K-major) and W^T rows of up to 8
//     taps x 32 channels [256 x 64] (B, K-major) into a two-stage ring;
//   * MMA warp: G[128 x 32*taps] = grad_y * W^T chunk by chunk of 64 output
//     channels into one of two TMEM accumulators (256 columns each);
//   * 8 epilogue warps (two per TMEM lane quarter, alternate taps): read G,
//     turn each 32x32 block so that a lane holds one channel, and add
//     G * m * w_corner into the window with shared-memory atomics (32 lanes on
//     32 consecutive words: no bank conflicts); at the end of the unit all of
//     them flush the window into grad_x and clear it.
// All waits are bounded; the records are the float32 sampling records of the
// data-backward pre-pass, W^T its transposed weights.
#include "kernels.h"
#include "tc_ptx.cuh"
#include "fwd_common.cuh"

namespace dcn {
namespace {

constexpr int GX_BM = 128;                  // pixels per unit (UMMA M)
constexpr int GX_SL = 32;                   // input channels per unit
constexpr int GX_BK = 64;                   // output channels per K chunk
constexpr int GX_TPG = 8;                   // taps per N group (N = 32 * taps <= 256)
constexpr int GX_EPI_WARPS = 8;
constexpr int GX_TMA_WARP = 8, GX_MMA_WARP = 9;
constexpr int GX_THREADS = 10 * 32;
constexpr int GX_STAGES = 2;
constexpr uint32_t GX_A_BYTES = GX_BM * GX_BK * 2;             // 16 KB
constexpr uint32_t GX_B_BYTES = GX_TPG * GX_SL * GX_BK * 2;    // 32 KB
constexpr int GX_TPITCH = 36;                                  // floats per row of a warp's 32x32 turn buffer
constexpr int GX_WIN_CELLS = 704;                              // window pixels (x 32 channels x 4 B = 88 KB)
constexpr int GX_MARGIN = 3;                                   // offset reach covered by the window, in rows

struct GxArgs {
    Shape s;
    const float4* rec;   // [G*K2][ppad]: {ly, lx, m, ((y0+1) << 16) | (x0+1)}, yx = ~0 when no neighbour is inside
    float* gx;
    unsigned* status;
    int ppad, nsl, ngroups, ctas;
    long long total_units;
};

__device__ __forceinline__ long long gx_unit_begin(int c, const GxArgs& a) { return a.total_units * c / a.ctas; }

// The window of the unit whose pixels start at p0: rows [r0, r0 + nr) of image
// b0, all W columns.
struct Window {
    int b0, r0, nr;
};
__device__ __forceinline__ Window unit_window(const Shape& s, int p0) {
    Window w;
    const int plane = s.Ho * s.Wo;
    w.b0 = p0 / plane;
    const int pl = min(min(p0 + GX_BM - 1, (w.b0 + 1) * plane - 1), s.P - 1);
    const int ho_lo = (p0 - w.b0 * plane) / s.Wo, ho_hi = (pl - w.b0 * plane) / s.Wo;
    int ra = ho_lo * s.stride - s.pad - GX_MARGIN;
    int rb = ho_hi * s.stride - s.pad + (s.K - 1) * s.dil + GX_MARGIN + 2;  // exclusive; +1 for the lower corner
    ra = max(ra, 0);
    rb = min(rb, s.H);
    const int cap = GX_WIN_CELLS / s.W;
    if (rb - ra > cap) {  // too tall: keep the middle rows (the others go straight to grad_x)
        const int cut = rb - ra - cap;
        ra += cut / 2;
        rb = ra + cap;
    }
    w.r0 = ra;
    w.nr = max(rb - ra, 0);
    return w;
}

__global__ void __launch_bounds__(GX_THREADS, 1)
    dcn_bwd_gx_kernel(const __grid_constant__ CUtensorMap tmap_dy, const __grid_constant__ CUtensorMap tmap_wt,
                      const GxArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Shape& s = a.s;
    constexpr uint32_t STAGE = GX_A_BYTES + GX_B_BYTES;
    float* win = reinterpret_cast<float*>(smem + GX_STAGES * STAGE);                  // [cells][32]
    float* turn = win + GX_WIN_CELLS * GX_SL;                                           // [8][32][TPITCH]
    uint64_t* bars = reinterpret_cast<uint64_t*>(turn + GX_EPI_WARPS * 32 * GX_TPITCH);
    uint64_t* full = bars;
    uint64_t* empty = bars + GX_STAGES;
    uint64_t* acc_full = empty + GX_STAGES;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* drain = acc_empty + 2;
    uint64_t* epi_bar = drain + 1;  // the epilogue warps' own barrier (bounded waits)
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(epi_bar + 1);
    volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
    const int kchunks = (s.Cout + GX_BK - 1) / GX_BK;

    if (threadIdx.x == 0) {
        for (int i = 0; i < GX_STAGES; ++i) {
            ptx::mbar_init(ptx::smem_u32(&full[i]), 1);
            ptx::mbar_init(ptx::smem_u32(&empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(ptx::smem_u32(&acc_full[i]), 1);
            ptx::mbar_init(ptx::smem_u32(&acc_empty[i]), GX_EPI_WARPS);
        }
        ptx::mbar_init(ptx::smem_u32(drain), 1);
        ptx::mbar_init(ptx::smem_u32(epi_bar), GX_EPI_WARPS);
        *s_abort = 0;
        ptx::fence_mbar_init();
    }
    for (int i = threadIdx.x; i < GX_WIN_CELLS * GX_SL / 4; i += GX_THREADS)
        reinterpret_cast<float4*>(win)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (warp == GX_MMA_WARP) {
        ptx::tmem_alloc(ptx::smem_u32(s_tmem), 512);
        ptx::tmem_relinquish();
    }
    if (warp == GX_TMA_WARP && lane == 0) {
        ptx::prefetch_tmap(&tmap_dy);
        ptx::prefetch_tmap(&tmap_wt);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *s_tmem;
    const long long ubeg = gx_unit_begin(blockIdx.x, a), uend = gx_unit_begin(blockIdx.x + 1, a);

    if (warp == GX_TMA_WARP) {
        // ------------------------------------------------- grad_y and W^T --
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, issued = 0, issued_par = 0;
            bool ok = true;
            for (long long u = ubeg; u < uend && ok; ++u) {
                const int mt = (int)(u / a.nsl), sl = (int)(u - (long long)mt * a.nsl);
                for (int j = 0; j < a.ngroups && ok; ++j) {
                    const int t0 = j * GX_TPG, nt = min(GX_TPG, s.K2 - t0);
                    for (int kc = 0; kc < kchunks; ++kc) {
                        if (!ptx::mbar_wait(ptx::smem_u32(&empty[stage]), phase ^ 1, s_abort, a.status, WAIT_LIMIT)) {
                            ok = false;
                            break;
                        }
                        uint8_t* st = smem + stage * STAGE;
                        const uint32_t fb = ptx::smem_u32(&full[stage]);
                        ptx::mbar_arrive_expect_tx(fb, GX_A_BYTES + (uint32_t)nt * GX_SL * GX_BK * 2);
                        ptx::tma_load_2d(ptx::smem_u32(st), &tmap_dy, fb, kc * GX_BK, mt * GX_BM);
                        for (int t = 0; t < nt; ++t)
                            ptx::tma_load_2d(ptx::smem_u32(st + GX_A_BYTES + t * GX_SL * 128), &tmap_wt, fb, kc * GX_BK,
                                             (t0 + t) * s.Cin + sl * GX_SL);
                        issued |= 1u << stage;
                        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
                        if (++stage == GX_STAGES) {
                            stage = 0;
                            phase ^= 1;
                        }
                    }
                }
            }
            if (*s_abort) {
                volatile int dummy = 0;
                for (int i = 0; i < GX_STAGES; ++i)
                    if ((issued >> i) & 1u)
                        ptx::mbar_wait(ptx::smem_u32(&full[i]), (issued_par >> i) & 1u, &dummy, nullptr, WAIT_LIMIT);
            }
        }
        __syncwarp();
    } else if (warp == GX_MMA_WARP) {
        // ----------------------------------------------------------- MMA --
        if (lane == 0) {
            int stage = 0, grp = 0;
            uint32_t phase = 0;
            const uint32_t s0 = ptx::smem_u32(smem);
            bool ok = true;
            for (long long u = ubeg; u < uend && ok; ++u) {
                for (int j = 0; j < a.ngroups && ok; ++j, ++grp) {
                    const int nt = min(GX_TPG, s.K2 - j * GX_TPG);
                    const uint32_t idesc = ptx::idesc_bf16_f32(GX_BM, GX_SL * nt);
                    const int abuf = grp & 1;
                    if (!ptx::mbar_wait(ptx::smem_u32(&acc_empty[abuf]), ((grp >> 1) & 1) ^ 1, s_abort, a.status,
                                        WAIT_LIMIT)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t d = tmem_base + (uint32_t)(abuf * 256);
                    for (int kc = 0; kc < kchunks; ++kc) {
                        if (!ptx::mbar_wait(ptx::smem_u32(&full[stage]), phase, s_abort, a.status, WAIT_LIMIT)) {
                            ok = false;
                            break;
                        }
                        ptx::tc_fence_after();
                        const uint32_t st = s0 + stage * STAGE;
#pragma unroll
                        for (int kk = 0; kk < GX_BK / 16; ++kk)
                            ptx::mma_bf16(d, ptx::sw128_desc(st + kk * 32), ptx::sw128_desc(st + GX_A_BYTES + kk * 32),
                                          idesc, (kc > 0 || kk > 0) ? 1u : 0u);
                        ptx::mma_commit(ptx::smem_u32(&empty[stage]));
                        if (++stage == GX_STAGES) {
                            stage = 0;
                            phase ^= 1;
                        }
                    }
                    if (!ok) break;
                    ptx::mma_commit(ptx::smem_u32(&acc_full[abuf]));
                }
            }
            ptx::mma_commit(ptx::smem_u32(drain));
            volatile int dummy = 0;
            ptx::mbar_wait(ptx::smem_u32(drain), 0, &dummy, a.status, WAIT_LIMIT);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ epilogue --
        const int quarter = warp & 3, half = warp >> 2;
        const int row = quarter * 32 + lane;
        const int plane = s.Ho * s.Wo;
        float* tb = turn + warp * 32 * GX_TPITCH;
        const uint32_t win_s = ptx::smem_u32(win);
        int grp = 0;
        uint32_t ephase = 0;
        bool ok = true;
        for (long long u = ubeg; u < uend && ok; ++u) {
            const int mt = (int)(u / a.nsl), sl = (int)(u - (long long)mt * a.nsl);
            const int g = sl * GX_SL / s.Cg;
            const int p0 = mt * GX_BM;
            const Window wd = unit_window(s, p0);
            const int p = p0 + row;
            const int bp = p < s.P ? p / plane : -1;
            const long long chan = (long long)sl * GX_SL + lane;  // this lane's channel within Cin
            for (int j = 0; j < a.ngroups && ok; ++j, ++grp) {
                const int t0 = j * GX_TPG, nt = min(GX_TPG, s.K2 - t0);
                const int abuf = grp & 1;
                if (!__all_sync(0xffffffffu, ptx::mbar_wait(ptx::smem_u32(&acc_full[abuf]), (grp >> 1) & 1, s_abort,
                                                            a.status, WAIT_LIMIT))) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                // this warp takes the group's taps of its parity
                float4 rc = make_float4(0.f, 0.f, 0.f, __uint_as_float(0xFFFFFFFFu));
                if (half < nt && p < s.P) rc = a.rec[(size_t)(g * s.K2 + t0 + half) * a.ppad + p];
                for (int t = half; t < nt; t += 2) {
                    float G[32];
                    ptx::tmem_ld32(tmem_base + (uint32_t)(abuf * 256 + t * GX_SL) + ((uint32_t)(quarter * 32) << 16), G);
                    const float4 cur = rc;
                    if (t + 2 < nt && p < s.P) rc = a.rec[(size_t)(g * s.K2 + t0 + t + 2) * a.ppad + p];
                    // this thread's sample: corner weights times m, corners inside the map / the window
                    const uint32_t yx = __float_as_uint(cur.w);
                    uint32_t flags = 0;  // bits 0-3: corner inside the map, 4-7: inside the window
                    int cell = 0;        // window cell of the top-left corner
                    long long gpix = 0;  // grad_x pixel index of the top-left corner
                    float w00 = 0.f, w01 = 0.f, w10 = 0.f, w11 = 0.f;
                    if (bp >= 0 && yx != 0xFFFFFFFFu) {
                        const int y0 = (int)(yx >> 16) - 1, x0 = (int)(yx & 0xFFFFu) - 1;
                        const float ly = cur.x, lx = cur.y, m = cur.z;
                        w00 = (1.f - ly) * (1.f - lx) * m;
                        w01 = (1.f - ly) * lx * m;
                        w10 = ly * (1.f - lx) * m;
                        w11 = ly * lx * m;
                        const bool xin0 = (unsigned)x0 < (unsigned)s.W, xin1 = (unsigned)(x0 + 1) < (unsigned)s.W;
                        const bool yin0 = (unsigned)y0 < (unsigned)s.H, yin1 = (unsigned)(y0 + 1) < (unsigned)s.H;
                        flags = (yin0 && xin0 ? 1u : 0u) | (yin0 && xin1 ? 2u : 0u) | (yin1 && xin0 ? 4u : 0u) |
                                (yin1 && xin1 ? 8u : 0u);
                        const bool inb = bp == wd.b0;
                        const bool wy0 = inb && y0 >= wd.r0 && y0 < wd.r0 + wd.nr;
                        const bool wy1 = inb && y0 + 1 >= wd.r0 && y0 + 1 < wd.r0 + wd.nr;
                        flags |= (((wy0 ? 3u : 0u) | (wy1 ? 12u : 0u)) & flags) << 4;
                        cell = (y0 - wd.r0) * s.W + x0;
                        gpix = ((long long)bp * s.H + y0) * s.W + x0;
                    }
                    // turn the 32x32 block: lane = channel, one pixel at a time
                    __syncwarp();
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        *reinterpret_cast<float4*>(tb + lane * GX_TPITCH + 4 * q) =
                            make_float4(G[4 * q], G[4 * q + 1], G[4 * q + 2], G[4 * q + 3]);
                    __syncwarp();
                    for (int i = 0; i < 32; ++i) {
                        const uint32_t fl = __shfl_sync(0xffffffffu, flags, i);
                        if (!fl) continue;  // warp-uniform
                        const float gv = tb[i * GX_TPITCH + lane];
                        const int ce = __shfl_sync(0xffffffffu, cell, i);
                        const float v00 = __shfl_sync(0xffffffffu, w00, i) * gv;
                        const float v01 = __shfl_sync(0xffffffffu, w01, i) * gv;
                        const float v10 = __shfl_sync(0xffffffffu, w10, i) * gv;
                        const float v11 = __shfl_sync(0xffffffffu, w11, i) * gv;
                        const uint32_t wa = win_s + (uint32_t)(ce * GX_SL + lane) * 4u;
                        const uint32_t rowb = (uint32_t)s.W * GX_SL * 4u;
                        if (fl & 0x10u) asm volatile("red.shared.add.f32 [%0], %1;" ::"r"(wa), "f"(v00) : "memory");
                        if (fl & 0x20u) asm volatile("red.shared.add.f32 [%0], %1;" ::"r"(wa + GX_SL * 4u), "f"(v01) : "memory");
                        if (fl & 0x40u) asm volatile("red.shared.add.f32 [%0], %1;" ::"r"(wa + rowb), "f"(v10) : "memory");
                        if (fl & 0x80u)
                            asm volatile("red.shared.add.f32 [%0], %1;" ::"r"(wa + rowb + GX_SL * 4u), "f"(v11) : "memory");
                        if ((fl & 0xFu) != (fl >> 4)) {
                            // corners inside the map but outside the window: straight to grad_x
                            const long long gp = __shfl_sync(0xffffffffu, gpix, i);
                            float* gb = a.gx + gp * s.Cin + chan;
                            const uint32_t direct = (fl & 0xFu) & ~(fl >> 4);
                            if (direct & 1u) atomicAdd(gb, v00);
                            if (direct & 2u) atomicAdd(gb + s.Cin, v01);
                            if (direct & 4u) atomicAdd(gb + (long long)s.W * s.Cin, v10);
                            if (direct & 8u) atomicAdd(gb + ((long long)s.W + 1) * s.Cin, v11);
                        }
                    }
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&acc_empty[abuf]));
            }
            if (!ok) break;
            // every epilogue warp is done with the unit: add the window into grad_x, clear it
            if (!epi_sync(epi_bar, ephase, s_abort, a.status)) {
                ok = false;
                break;
            }
            const int cells = wd.nr * s.W;
            const int et = threadIdx.x;  // 0 .. 255
            for (int c = et >> 3; c < cells; c += GX_EPI_WARPS * 32 / 8) {
                float4* wp = reinterpret_cast<float4*>(win + c * GX_SL) + (et & 7);
                const float4 v = *wp;
                if (v.x != 0.f || v.y != 0.f || v.z != 0.f || v.w != 0.f) {
                    const long long pix = ((long long)wd.b0 * s.H + wd.r0) * s.W + c;
                    ptx::red_add_v4(a.gx + pix * s.Cin + (long long)sl * GX_SL + 4 * (et & 7), v.x, v.y, v.z, v.w);
                    *wp = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
            if (!epi_sync(epi_bar, ephase, s_abort, a.status)) {
                ok = false;
                break;
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == GX_MMA_WARP) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, 512);
    }
}

uint32_t gx_smem_bytes() {
    return GX_STAGES * (GX_A_BYTES + GX_B_BYTES) + GX_WIN_CELLS * GX_SL * 4 + GX_EPI_WARPS * 32 * GX_TPITCH * 4 +
           (4 * GX_STAGES + 9) * 8 + 16 + 1024;
}

bool encode_kmajor_rows(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
    auto encode = get_encode();
    if (!encode) return false;
    cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)inner * 2};
    cuuint32_t box[2] = {(cuuint32_t)GX_BK, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// Groups of whole 32-channel slices, rows of W short enough for 32-bit pixel
// indexing; the data-backward pre-pass supplies the records and W^T.
bool bwd_gx_supported(const Shape& s) {
    return s.Cg % GX_SL == 0 && s.Cout % 8 == 0 && s.Cin % 8 == 0 && s.W <= GX_WIN_CELLS &&
           gx_smem_bytes() <= 227 * 1024;
}

cudaError_t bwd_gx_tc(const Shape& s, const void* gy, const void* wt, const void* rec, int ppad, float* gx,
                      unsigned* status, cudaStream_t st, int* launches) {
    if (!bwd_gx_supported(s)) return cudaErrorInvalidValue;
    CUtensorMap map_dy, map_wt;
    if (!encode_kmajor_rows(&map_dy, gy, (uint64_t)s.Cout, (uint64_t)s.P, GX_BM) ||
        !encode_kmajor_rows(&map_wt, wt, (uint64_t)s.Cout, (uint64_t)s.KC, GX_SL))
        return cudaErrorInvalidValue;
    static DeviceFlags attr;
    cudaError_t e = max_dynamic_smem_once((const void*)dcn_bwd_gx_kernel, 227 * 1024, attr);
    if (e != cudaSuccess) return e;
    GxArgs a;
    a.s = s;
    a.rec = reinterpret_cast<const float4*>(rec);
    a.gx = gx;
    a.status = status;
    a.ppad = ppad;
    a.nsl = s.Cin / GX_SL;
    a.ngroups = (s.K2 + GX_TPG - 1) / GX_TPG;
    const int m_tiles = (s.P + GX_BM - 1) / GX_BM;
    a.total_units = (long long)m_tiles * a.nsl;
    a.ctas = (int)std::min<long long>(num_sms(), a.total_units);
    dcn_bwd_gx_kernel<<<a.ctas, GX_THREADS, gx_smem_bytes(), st>>>(map_dy, map_wt, a);
    if (launches) *launches += 1;
    return cudaGetLastError();
}

}  // namespace dcn
