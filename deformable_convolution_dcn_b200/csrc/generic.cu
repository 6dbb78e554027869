// Generic CUDA-core kernels of libdcn_b200: every shape, float32 or bfloat16
// inputs, float32 arithmetic. They serve shapes the specialised kernels do not
// take (channel counts that are not multiples of 8, for instance) and are the
// first GPU path of each pass. Work is tiled through shared memory: the
// deformable gather fills a tile of modulated samples ("columns") that never
// leaves the SM, and a register-blocked FMA loop contracts it with the weight.
#include "common.cuh"
#include "kernels.h"

namespace dcn {

// ---------------------------------------------------------------- forward --
// Block: 64 output pixels x 64 output channels, 256 threads, 4x4 outputs each.
// K loop over (tap, channel) in chunks of 16 in the weight's [K*K*Cin] order.
template <typename T>
__global__ void __launch_bounds__(256) generic_forward_kernel(Shape s, const T* __restrict__ x,
                                                              const T* __restrict__ off, const T* __restrict__ mask,
                                                              const T* __restrict__ w, const T* __restrict__ bias,
                                                              T* __restrict__ y) {
    constexpr int BP = 64, BO = 64, KCH = 16;
    __shared__ float As[KCH][BP + 4];
    __shared__ float Bs[KCH][BO + 4];
    const int p0 = blockIdx.x * BP, o0 = blockIdx.y * BO;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[a][e] = 0.f;

    for (int k0 = 0; k0 < s.KC; k0 += KCH) {
        for (int e = tid; e < BP * KCH; e += 256) {
            int kk = e / BP, px = e - (e / BP) * BP;
            int kc = k0 + kk, p = p0 + px;
            float v = 0.f;
            if (kc < s.KC && p < s.P) {
                int tap = kc / s.Cin, c = kc - tap * s.Cin;
                TapSample t = tap_sample(s, off, mask, p, c / s.Cg, tap);
                v = t.m * bilinear_at(s, x, t, c);
            }
            As[kk][px] = v;
        }
        for (int e = tid; e < BO * KCH; e += 256) {
            int kk = e % KCH, o = e / KCH;
            int kc = k0 + kk;
            Bs[kk][o] = (kc < s.KC && o0 + o < s.Cout) ? ldf(w + (size_t)(o0 + o) * s.KC + kc) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < KCH; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) a[u] = As[kk][ty * 4 + u];
#pragma unroll
            for (int u = 0; u < 4; ++u) b[u] = Bs[kk][tx * 4 + u];
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(a[u], b[v], acc[u][v]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        int p = p0 + ty * 4 + u;
        if (p >= s.P) continue;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            int o = o0 + tx * 4 + v;
            if (o >= s.Cout) continue;
            float r = acc[u][v] + (bias ? ldf(bias + o) : 0.f);
            y[(size_t)p * s.Cout + o] = from_float<T>(r);
        }
    }
}

// ------------------------------------------------------------ backward data --
// Block: 64 output pixels of one (group, tap). For each chunk of 32 channels of
// the group: gcol[p, c] = sum_o grad_y[p, o] * w[o, tap, c] through shared
// tiles, then one warp per pixel walks the 32 channels: it scatters
// gcol * m * (neighbour weight) into grad_x with atomics and accumulates the
// offset and mask gradients, which the block owns and writes once.
template <typename T>
__global__ void __launch_bounds__(256) generic_backward_data_kernel(Shape s, const T* __restrict__ x,
                                                                    const T* __restrict__ off,
                                                                    const T* __restrict__ mask,
                                                                    const T* __restrict__ w,
                                                                    const T* __restrict__ gy, float* __restrict__ gx,
                                                                    float* __restrict__ goff,
                                                                    float* __restrict__ gmask) {
    constexpr int BP = 64, BC = 32, KO = 16;
    __shared__ float Ys[KO][BP + 1];
    __shared__ float Ws[KO][BC + 1];
    __shared__ float Gs[BP][BC + 1];
    __shared__ TapSample ts[BP];
    __shared__ float r_dy[BP], r_dx[BP], r_m[BP];
    const int p0 = blockIdx.x * BP;
    const int g = blockIdx.y / s.K2, tap = blockIdx.y - (blockIdx.y / s.K2) * s.K2;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid < BP) {
        int p = p0 + tid;
        if (p < s.P) ts[tid] = tap_sample(s, off, mask, p, g, tap);
        r_dy[tid] = r_dx[tid] = r_m[tid] = 0.f;
    }
    __syncthreads();
    const int tx = tid & 7, ty = tid >> 3;  // 4 channels x 2 pixels per thread in the contraction
    for (int c0 = 0; c0 < s.Cg; c0 += BC) {
        float acc[2][4];
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[a][e] = 0.f;
        for (int o0 = 0; o0 < s.Cout; o0 += KO) {
            for (int e = tid; e < BP * KO; e += 256) {
                int px = e / KO, ko = e - (e / KO) * KO;
                int p = p0 + px, o = o0 + ko;
                Ys[ko][px] = (p < s.P && o < s.Cout) ? ldf(gy + (size_t)p * s.Cout + o) : 0.f;
            }
            for (int e = tid; e < KO * BC; e += 256) {
                int ko = e / BC, c = e - (e / BC) * BC;
                int o = o0 + ko, cc = c0 + c;
                Ws[ko][c] = (o < s.Cout && cc < s.Cg)
                                ? ldf(w + (size_t)o * s.KC + (size_t)tap * s.Cin + g * s.Cg + cc)
                                : 0.f;
            }
            __syncthreads();
#pragma unroll
            for (int ko = 0; ko < KO; ++ko) {
                float a0 = Ys[ko][ty * 2], a1 = Ys[ko][ty * 2 + 1];
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    float b = Ws[ko][tx * 4 + v];
                    acc[0][v] = fmaf(a0, b, acc[0][v]);
                    acc[1][v] = fmaf(a1, b, acc[1][v]);
                }
            }
            __syncthreads();
        }
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int v = 0; v < 4; ++v) Gs[ty * 2 + u][tx * 4 + v] = acc[u][v];
        __syncthreads();
        for (int px = warp; px < BP; px += 8) {
            int p = p0 + px, c = c0 + lane;
            float pdy = 0.f, pdx = 0.f, pm = 0.f;
            if (p < s.P && c < s.Cg) {
                const TapSample t = ts[px];
                const float G = Gs[px][lane];
                const int ch = g * s.Cg + c;
                const size_t img = (size_t)t.b * s.H * s.W;
                const bool i00 = inside(s, t.y0, t.x0), i01 = inside(s, t.y0, t.x0 + 1);
                const bool i10 = inside(s, t.y0 + 1, t.x0), i11 = inside(s, t.y0 + 1, t.x0 + 1);
                const size_t a00 = (img + (size_t)t.y0 * s.W + t.x0) * s.Cin + ch;
                const size_t a01 = a00 + s.Cin, a10 = a00 + (size_t)s.W * s.Cin, a11 = a10 + s.Cin;
                float v00 = i00 ? ldf(x + a00) : 0.f, v01 = i01 ? ldf(x + a01) : 0.f;
                float v10 = i10 ? ldf(x + a10) : 0.f, v11 = i11 ? ldf(x + a11) : 0.f;
                float w00 = (1.f - t.ly) * (1.f - t.lx), w01 = (1.f - t.ly) * t.lx;
                float w10 = t.ly * (1.f - t.lx), w11 = t.ly * t.lx;
                float val = w00 * v00 + w01 * v01 + w10 * v10 + w11 * v11;
                float dpy = (1.f - t.lx) * (v10 - v00) + t.lx * (v11 - v01);
                float dpx = (1.f - t.ly) * (v01 - v00) + t.ly * (v11 - v10);
                float gm = G * t.m;
                pm = G * val;
                pdy = gm * dpy;
                pdx = gm * dpx;
                if (gx) {
                    if (i00) atomicAdd(gx + a00, gm * w00);
                    if (i01) atomicAdd(gx + a01, gm * w01);
                    if (i10) atomicAdd(gx + a10, gm * w10);
                    if (i11) atomicAdd(gx + a11, gm * w11);
                }
            }
#pragma unroll
            for (int sh = 16; sh > 0; sh >>= 1) {
                pdy += __shfl_xor_sync(0xffffffffu, pdy, sh);
                pdx += __shfl_xor_sync(0xffffffffu, pdx, sh);
                pm += __shfl_xor_sync(0xffffffffu, pm, sh);
            }
            if (lane == 0) {
                r_dy[px] += pdy;
                r_dx[px] += pdx;
                r_m[px] += pm;
            }
        }
        __syncthreads();
    }
    if (tid < BP) {
        int p = p0 + tid;
        if (p < s.P) {
            int plane = s.Ho * s.Wo, b = p / plane, pix = p - b * plane;
            if (goff) {
                size_t ob = ((size_t)b * 2 * s.G * s.K2 + (size_t)g * 2 * s.K2 + 2 * tap) * plane + pix;
                goff[ob] = r_dy[tid];
                goff[ob + plane] = r_dx[tid];
            }
            if (gmask) gmask[((size_t)b * s.G * s.K2 + (size_t)g * s.K2 + tap) * plane + pix] = r_m[tid];
        }
    }
}

// ---------------------------------------------------------- backward weight --
// Block: 64 output channels x 64 (tap, channel) columns over one slice of the
// output pixels; the column tile is regenerated by the gather. Partial sums go
// to grad_weight with atomics (grad_weight is zeroed first).
template <typename T>
__global__ void __launch_bounds__(256) generic_backward_weight_kernel(Shape s, const T* __restrict__ x,
                                                                      const T* __restrict__ off,
                                                                      const T* __restrict__ mask,
                                                                      const T* __restrict__ gy,
                                                                      float* __restrict__ gw, int pix_per_split) {
    constexpr int BO = 64, BK = 64, PC = 16;
    __shared__ float Ys[PC][BO + 4];
    __shared__ float Cs[PC][BK + 4];
    const int k0 = blockIdx.x * BK, o0 = blockIdx.y * BO;
    const int pbeg = blockIdx.z * pix_per_split;
    const int pend = min(s.P, pbeg + pix_per_split);
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[a][e] = 0.f;
    for (int pc = pbeg; pc < pend; pc += PC) {
        for (int e = tid; e < PC * BO; e += 256) {
            int pp = e / BO, o = e - (e / BO) * BO;
            int p = pc + pp;
            Ys[pp][o] = (p < pend && o0 + o < s.Cout) ? ldf(gy + (size_t)p * s.Cout + o0 + o) : 0.f;
        }
        for (int e = tid; e < PC * BK; e += 256) {
            int kk = e / PC, pp = e - (e / PC) * PC;
            int p = pc + pp, kc = k0 + kk;
            float v = 0.f;
            if (p < pend && kc < s.KC) {
                int tap = kc / s.Cin, c = kc - tap * s.Cin;
                TapSample t = tap_sample(s, off, mask, p, c / s.Cg, tap);
                v = t.m * bilinear_at(s, x, t, c);
            }
            Cs[pp][kk] = v;
        }
        __syncthreads();
#pragma unroll
        for (int pp = 0; pp < PC; ++pp) {
            float a[4], b[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) a[u] = Ys[pp][ty * 4 + u];
#pragma unroll
            for (int u = 0; u < 4; ++u) b[u] = Cs[pp][tx * 4 + u];
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(a[u], b[v], acc[u][v]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        int o = o0 + ty * 4 + u;
        if (o >= s.Cout) continue;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            int kc = k0 + tx * 4 + v;
            if (kc < s.KC) atomicAdd(gw + (size_t)o * s.KC + kc, acc[u][v]);
        }
    }
}

// grad_bias[o] = sum_p grad_y[p, o]: one thread per channel and 64-pixel slice
// (loads coalesced across the channels of a warp, eight in flight per thread),
// one atomic per thread.
template <typename T>
__global__ void __launch_bounds__(256) bias_grad_kernel(Shape s, const T* __restrict__ gy, float* __restrict__ gb,
                                                        int pix_per_split) {
    const int o = blockIdx.x * blockDim.x + threadIdx.x;
    if (o >= s.Cout) return;
    const int pbeg = blockIdx.y * pix_per_split, pend = min(s.P, pbeg + pix_per_split);
    float acc = 0.f;
    for (int p = pbeg; p < pend; p += 8) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = (p + u < pend) ? ldf(gy + (size_t)(p + u) * s.Cout + o) : 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) acc += v[u];
    }
    atomicAdd(gb + o, acc);
}

// grad_bias with 16-byte loads: a block takes a slice of pixels; its threads
// form rows x groups, each thread one group of V = 16 / sizeof(T) channels and
// every rows-th pixel of the slice; the rows are summed in shared memory and
// one atomic per channel and block adds the slice into grad_bias.
template <typename T>
__global__ void __launch_bounds__(256) bias_grad_vec_kernel(Shape s, const T* __restrict__ gy, float* __restrict__ gb,
                                                            int pix_per_block) {
    constexpr int V = 16 / (int)sizeof(T);
    __shared__ float red[256 * V];
    const int groups = s.Cout / V, rows = 256 / groups;
    const int t = threadIdx.x, g = t % groups, pr = t / groups;
    const int pbeg = blockIdx.x * pix_per_block, pend = min(s.P, pbeg + pix_per_block);
    float acc[V];
#pragma unroll
    for (int v = 0; v < V; ++v) acc[v] = 0.f;
    if (pr < rows) {
        // eight pixels' loads in flight before any is summed (a missing pixel reads as zero)
        constexpr int BATCH = 8;
        for (int p0 = pbeg + pr; p0 < pend; p0 += BATCH * rows) {
            uint4 qs[BATCH];
#pragma unroll
            for (int u = 0; u < BATCH; ++u) {
                const int p = p0 + u * rows;
                qs[u] = p < pend ? __ldg(reinterpret_cast<const uint4*>(gy + (size_t)p * s.Cout) + g)
                                 : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < BATCH; ++u) {
                const uint4 q = qs[u];
                if constexpr (sizeof(T) == 2) {
                    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        acc[2 * i] += __uint_as_float(w[i] << 16);
                        acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
                    }
                } else {
                    acc[0] += __uint_as_float(q.x);
                    acc[1] += __uint_as_float(q.y);
                    acc[2] += __uint_as_float(q.z);
                    acc[3] += __uint_as_float(q.w);
                }
            }
        }
#pragma unroll
        for (int v = 0; v < V; ++v) red[pr * s.Cout + g * V + v] = acc[v];
    }
    __syncthreads();
    for (int o = t; o < s.Cout; o += 256) {
        float sum = 0.f;
        for (int r = 0; r < rows; ++r) sum += red[r * s.Cout + o];
        atomicAdd(gb + o, sum);
    }
}

// ------------------------------------------------------------- launchers --

static int splits_for(int P, int tiles, int per_block_min) {
    // enough pixel slices to give the grid a few waves over 148 SMs
    int want = (4 * 148 + tiles - 1) / tiles;
    int maxs = (P + per_block_min - 1) / per_block_min;
    return want < 1 ? 1 : (want > maxs ? maxs : want);
}

template <typename T>
static cudaError_t launch_generic_forward(const Shape& s, const void* x, const void* off, const void* mask,
                                          const void* w, const void* bias, void* y, cudaStream_t st) {
    dim3 grid((s.P + 63) / 64, (s.Cout + 63) / 64);
    generic_forward_kernel<T><<<grid, 256, 0, st>>>(s, (const T*)x, (const T*)off, (const T*)mask, (const T*)w,
                                                    (const T*)bias, (T*)y);
    return cudaGetLastError();
}

cudaError_t generic_forward(const Shape& s, int dtype, const void* x, const void* off, const void* mask,
                            const void* w, const void* bias, void* y, cudaStream_t st) {
    return dtype == 0 ? launch_generic_forward<float>(s, x, off, mask, w, bias, y, st)
                      : launch_generic_forward<bf16>(s, x, off, mask, w, bias, y, st);
}

template <typename T>
static cudaError_t launch_generic_backward_data(const Shape& s, const void* x, const void* off, const void* mask,
                                                const void* w, const void* gy, float* gx, float* goff,
                                                float* gmask, cudaStream_t st) {
    dim3 grid((s.P + 63) / 64, s.G * s.K2);
    generic_backward_data_kernel<T><<<grid, 256, 0, st>>>(s, (const T*)x, (const T*)off, (const T*)mask,
                                                          (const T*)w, (const T*)gy, gx, goff, gmask);
    return cudaGetLastError();
}

cudaError_t generic_backward_data(const Shape& s, int dtype, const void* x, const void* off, const void* mask,
                                  const void* w, const void* gy, float* gx, float* goff, float* gmask,
                                  cudaStream_t st) {
    return dtype == 0 ? launch_generic_backward_data<float>(s, x, off, mask, w, gy, gx, goff, gmask, st)
                      : launch_generic_backward_data<bf16>(s, x, off, mask, w, gy, gx, goff, gmask, st);
}

template <typename T>
static cudaError_t launch_generic_backward_weight(const Shape& s, const void* x, const void* off, const void* mask,
                                                  const void* gy, float* gw, cudaStream_t st) {
    int tiles = ((s.KC + 63) / 64) * ((s.Cout + 63) / 64);
    int splits = splits_for(s.P, tiles, 256);
    int per = (s.P + splits - 1) / splits;
    per = (per + 15) / 16 * 16;
    splits = (s.P + per - 1) / per;
    dim3 grid((s.KC + 63) / 64, (s.Cout + 63) / 64, splits);
    generic_backward_weight_kernel<T><<<grid, 256, 0, st>>>(s, (const T*)x, (const T*)off, (const T*)mask,
                                                            (const T*)gy, gw, per);
    return cudaGetLastError();
}

cudaError_t generic_backward_weight(const Shape& s, int dtype, const void* x, const void* off, const void* mask,
                                    const void* gy, float* gw, cudaStream_t st) {
    return dtype == 0 ? launch_generic_backward_weight<float>(s, x, off, mask, gy, gw, st)
                      : launch_generic_backward_weight<bf16>(s, x, off, mask, gy, gw, st);
}

cudaError_t bias_grad(const Shape& s, int dtype, const void* gy, float* gb, cudaStream_t st, bool pdl) {
    const int esz = dtype == 0 ? 4 : 2, V = 16 / esz;
    if ((reinterpret_cast<uintptr_t>(gy) & 15) == 0 && s.Cout % V == 0 && s.Cout / V <= 256 && s.P > 0) {
        const int blocks = std::min<long long>(2 * 148, s.P);
        const int per_block = (int)((s.P + blocks - 1) / blocks);
        const int nb = (int)((s.P + per_block - 1) / per_block);
        // pdl: a programmatic dependent of the kernel before it, which neither writes
        // grad_y nor reads grad_bias (the weight kernel): it may run alongside it
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)nb);
        cfg.blockDim = dim3(256);
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = pdl ? 1 : 0;
        if (dtype == 0) return cudaLaunchKernelEx(&cfg, bias_grad_vec_kernel<float>, s, (const float*)gy, gb, per_block);
        return cudaLaunchKernelEx(&cfg, bias_grad_vec_kernel<bf16>, s, (const bf16*)gy, gb, per_block);
    }
    const int per = 64;
    dim3 g2((s.Cout + 255) / 256, (s.P + per - 1) / per);
    if (dtype == 0)
        bias_grad_kernel<float><<<g2, 256, 0, st>>>(s, (const float*)gy, gb, per);
    else
        bias_grad_kernel<bf16><<<g2, 256, 0, st>>>(s, (const bf16*)gy, gb, per);
    return cudaGetLastError();
}

}  // namespace dcn
