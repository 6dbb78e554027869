// (Modulated) deformable RoI pooling, forward and backward (notes, "可变形ROI
// pooling": a RoI of w x h is cut into k x k bins, each output averages the
// pixels of its bin; the deformable form moves every bin by an offset given as
// a fraction of the RoI's width and height, read by bilinear interpolation;
// DCNv2 section 3.2: a modulation scalar per bin).
//
//   roi r = (b, x1, y1, x2, y2), h = max(y2 - y1, 0), w = max(x2 - x1, 0);
//   bin t = i*k + j holds the integer offsets (u, v), floor(i*h/k) <= u <
//   ceil((i+1)*h/k) and likewise v with w, n of them;
//   y[r][i][j][c] = m / n * sum over (u, v) of x_b(y1 + u + dy, x1 + v + dx, c),
//   (dy, dx) = gamma * (off[r][2t] * h, off[r][2t+1] * w), m = mask[r][t] or 1,
//   bilinear with neighbours outside the map contributing zero; 0 for an empty
//   bin or a batch index outside [0, B).
//
// One block per (RoI, bin), threads over channels (NHWC: consecutive threads
// read consecutive 16-byte channel vectors of one neighbour; one channel per
// thread when C is not a multiple of 16 bytes). Samples whose bilinear footprint
// misses the map contribute exactly zero, so the sample loops run only over the
// rows and columns that can touch it, which also bounds them for any RoI size;
// n still counts the whole bin. The backward scatters grad_x with float atomics
// and reduces the bin's offset and mask gradients over its channels in a fixed
// order in shared memory (no atomics).
#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace dcn {
namespace {

struct BinGeom {
    int b;             // batch index, -1 when outside [0, B)
    float y1, x1, h, w;
    float dy, dx, m;
    float n;           // samples in the bin (the divisor)
    int u_lo, u_hi, v_lo, v_hi;  // sample rows / columns that can touch the map
};

template <typename T>
__device__ __forceinline__ BinGeom bin_geom(const RoiArgs& a, const T* off, const T* mask, int r, int t) {
    BinGeom g;
    const float* roi = a.rois + (size_t)r * 5;
    // the batch index is the RoI's first value truncated toward zero; outside [0, B) the RoI pools to zeros
    g.b = (roi[0] > -1.f && roi[0] < (float)a.B) ? (int)roi[0] : -1;
    g.x1 = roi[1];
    g.y1 = roi[2];
    g.h = fmaxf(roi[4] - roi[2], 0.f);
    g.w = fmaxf(roi[3] - roi[1], 0.f);
    const int i = t / a.k, j = t - i * a.k;
    const float fu0 = floorf(i * g.h / a.k), fu1 = ceilf((i + 1) * g.h / a.k);
    const float fv0 = floorf(j * g.w / a.k), fv1 = ceilf((j + 1) * g.w / a.k);
    g.n = (fu1 - fu0) * (fv1 - fv0);
    const int kk = a.k * a.k;
    g.dy = off ? a.gamma * ldf(off + (size_t)r * 2 * kk + 2 * t) * g.h : 0.f;
    g.dx = off ? a.gamma * ldf(off + (size_t)r * 2 * kk + 2 * t + 1) * g.w : 0.f;
    g.m = mask ? ldf(mask + (size_t)r * kk + t) : 1.f;
    // rows u with y1 + u + dy in (-1, H) (a sample at -1 or H exactly adds zero), clamped before conversion
    const float lim = 1073741824.f;
    const float ulo = fmaxf(fu0, floorf(-1.f - g.y1 - g.dy)), uhi = fminf(fu1, ceilf((float)a.H - g.y1 - g.dy) + 1.f);
    const float vlo = fmaxf(fv0, floorf(-1.f - g.x1 - g.dx)), vhi = fminf(fv1, ceilf((float)a.W - g.x1 - g.dx) + 1.f);
    g.u_lo = (int)fminf(fmaxf(ulo, -lim), lim);
    g.u_hi = (int)fminf(fmaxf(uhi, -lim), lim);
    g.v_lo = (int)fminf(fmaxf(vlo, -lim), lim);
    g.v_hi = (int)fminf(fmaxf(vhi, -lim), lim);
    if (!(g.n > 0.f)) g.b = -1;
    return g;
}

struct Corner {
    int y0, x0;
    float ly, lx;
};

__device__ __forceinline__ Corner corner(float py, float px) {
    Corner c;
    const float fy = floorf(py), fx = floorf(px);
    c.y0 = (int)fy;
    c.x0 = (int)fx;
    c.ly = py - fy;
    c.lx = px - fx;
    return c;
}

template <typename T>
__device__ __forceinline__ float px_or_zero(const T* xb, const RoiArgs& a, int r, int q, int c) {
    if (r < 0 || r >= a.H || q < 0 || q >= a.W) return 0.f;
    return ldf(xb + ((size_t)r * a.W + q) * a.C + c);
}

// A bin's samples sit on a unit grid (rows y1 + dy + u, columns x1 + dx + v):
// all share the fractions (ly, lx), and sample u's bilinear rows are
// fy + u and fy + u + 1. Summed over the bin, the pixel rows fy + u_lo + a,
// a = 0 .. nu (nu = the number of sample rows), weigh wy(a) = 1 - ly for the
// first, ly for the last, 1 in between (and likewise the columns), so the bin
// reads each of its (nu + 1) x (nv + 1) pixels once instead of four times per
// sample. Sample positions are taken from the bin's first row and column.
struct BinBox {
    int y0, x0;   // top-left pixel of the box (may lie outside the map)
    int nu, nv;   // sample rows and columns (the box is (nu + 1) x (nv + 1) pixels)
    float ly, lx;
};
__device__ __forceinline__ BinBox bin_box(const BinGeom& g) {
    BinBox bx;
    const Corner q = corner(g.y1 + g.u_lo + g.dy, g.x1 + g.v_lo + g.dx);
    bx.y0 = q.y0;
    bx.x0 = q.x0;
    bx.ly = q.ly;
    bx.lx = q.lx;
    bx.nu = max(g.u_hi - g.u_lo, 0);
    bx.nv = max(g.v_hi - g.v_lo, 0);
    return bx;
}
// the box weight of pixel row a (0 .. n) for n sample rows with fraction l
__device__ __forceinline__ float box_w(int a, int n, float l) {
    return (a < n ? 1.f - l : 0.f) + (a > 0 ? l : 0.f);
}

template <typename T>
__global__ void __launch_bounds__(256) droi_fwd_kernel(RoiArgs a, const T* __restrict__ x, const T* __restrict__ off,
                                                       const T* __restrict__ mask, T* __restrict__ y) {
    const int bin = blockIdx.x, kk = a.k * a.k;
    const int r = bin / kk, t = bin - r * kk;
    const BinGeom g = bin_geom(a, off, mask, r, t);
    T* yb = y + (size_t)bin * a.C;
    if (g.b < 0) {
        for (int c = threadIdx.x; c < a.C; c += blockDim.x) yb[c] = from_float<T>(0.f);
        return;
    }
    const T* xb = x + (size_t)g.b * a.H * a.W * a.C;
    for (int c = threadIdx.x; c < a.C; c += blockDim.x) {
        float acc = 0.f;
        for (int u = g.u_lo; u < g.u_hi; ++u)
            for (int v = g.v_lo; v < g.v_hi; ++v) {
                const Corner q = corner(g.y1 + u + g.dy, g.x1 + v + g.dx);
                acc += (1.f - q.ly) * ((1.f - q.lx) * px_or_zero(xb, a, q.y0, q.x0, c) +
                                       q.lx * px_or_zero(xb, a, q.y0, q.x0 + 1, c)) +
                       q.ly * ((1.f - q.lx) * px_or_zero(xb, a, q.y0 + 1, q.x0, c) +
                               q.lx * px_or_zero(xb, a, q.y0 + 1, q.x0 + 1, c));
            }
        yb[c] = from_float<T>(g.m * acc / g.n);
    }
}

// 16 bytes of channels: 8 bf16 or 4 float32, widened to float
template <typename T>
struct Vec16 {
    static constexpr int N = 16 / sizeof(T);
};

template <typename T>
__device__ __forceinline__ void load16(const T* p, float (&v)[Vec16<T>::N]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[q]));
            v[2 * q] = f.x;
            v[2 * q + 1] = f.y;
        }
    } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) v[q] = __uint_as_float(w[q]);
    }
}

template <typename T>
__device__ __forceinline__ void store16(T* p, const float (&v)[Vec16<T>::N]) {
    uint32_t w[4];
    if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
            w[q] = *reinterpret_cast<const uint32_t*>(&h);
        }
    } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) w[q] = __float_as_uint(v[q]);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

// As droi_fwd_kernel, 16 bytes of channels per thread (C a multiple of 16 bytes, x and y 16-byte aligned).
template <typename T>
__global__ void __launch_bounds__(256) droi_fwd_vec_kernel(RoiArgs a, const T* __restrict__ x,
                                                           const T* __restrict__ off, const T* __restrict__ mask,
                                                           T* __restrict__ y) {
    constexpr int N = Vec16<T>::N;
    const int bin = blockIdx.x, kk = a.k * a.k;
    const int r = bin / kk, t = bin - r * kk;
    const BinGeom g = bin_geom(a, off, mask, r, t);
    T* yb = y + (size_t)bin * a.C;
    const int nv = a.C / N;
    if (g.b < 0) {
        float z[N];
#pragma unroll
        for (int e = 0; e < N; ++e) z[e] = 0.f;
        for (int cv = threadIdx.x; cv < nv; cv += blockDim.x) store16(yb + cv * N, z);
        return;
    }
    const T* xb = x + (size_t)g.b * a.H * a.W * a.C;
    const BinBox bx = bin_box(g);
    for (int cv = threadIdx.x; cv < nv; cv += blockDim.x) {
        const int c = cv * N;
        float acc[N];
#pragma unroll
        for (int e = 0; e < N; ++e) acc[e] = 0.f;
        if (bx.nu > 0 && bx.nv > 0)
            for (int ra = 0; ra <= bx.nu; ++ra) {
                const int rr = bx.y0 + ra;
                if (rr < 0 || rr >= a.H) continue;
                const float wy = box_w(ra, bx.nu, bx.ly);
                for (int cb = 0; cb <= bx.nv; ++cb) {
                    const int cc = bx.x0 + cb;
                    if (cc < 0 || cc >= a.W) continue;
                    const float wt = wy * box_w(cb, bx.nv, bx.lx);
                    float vv[N];
                    load16(xb + ((size_t)rr * a.W + cc) * a.C + c, vv);
#pragma unroll
                    for (int e = 0; e < N; ++e) acc[e] += wt * vv[e];
                }
            }
        const float sc = g.m / g.n;
#pragma unroll
        for (int e = 0; e < N; ++e) acc[e] *= sc;
        store16(yb + c, acc);
    }
}

__device__ __forceinline__ void add_if_inside(float* gxb, const RoiArgs& a, int r, int q, int c, float v) {
    if (r < 0 || r >= a.H || q < 0 || q >= a.W) return;
    atomicAdd(gxb + ((size_t)r * a.W + q) * a.C + c, v);
}

template <typename T>
__global__ void __launch_bounds__(256) droi_bwd_kernel(RoiArgs a, const T* __restrict__ x, const T* __restrict__ off,
                                                       const T* __restrict__ mask, const T* __restrict__ gy,
                                                       float* __restrict__ gx, float* __restrict__ goff,
                                                       float* __restrict__ gmask) {
    __shared__ float red[3][256];
    const int bin = blockIdx.x, kk = a.k * a.k;
    const int r = bin / kk, t = bin - r * kk;
    const BinGeom g = bin_geom(a, off, mask, r, t);
    float s_dy = 0.f, s_dx = 0.f, s_m = 0.f;
    if (g.b >= 0) {
        const T* xb = x + (size_t)g.b * a.H * a.W * a.C;
        float* gxb = gx + (size_t)g.b * a.H * a.W * a.C;
        const T* gyb = gy + (size_t)bin * a.C;
        for (int c = threadIdx.x; c < a.C; c += blockDim.x) {
            const float gc = ldf(gyb + c) / g.n;
            const float gm = gc * g.m;
            for (int u = g.u_lo; u < g.u_hi; ++u)
                for (int v = g.v_lo; v < g.v_hi; ++v) {
                    const Corner q = corner(g.y1 + u + g.dy, g.x1 + v + g.dx);
                    const float v00 = px_or_zero(xb, a, q.y0, q.x0, c), v01 = px_or_zero(xb, a, q.y0, q.x0 + 1, c);
                    const float v10 = px_or_zero(xb, a, q.y0 + 1, q.x0, c);
                    const float v11 = px_or_zero(xb, a, q.y0 + 1, q.x0 + 1, c);
                    add_if_inside(gxb, a, q.y0, q.x0, c, gm * (1.f - q.ly) * (1.f - q.lx));
                    add_if_inside(gxb, a, q.y0, q.x0 + 1, c, gm * (1.f - q.ly) * q.lx);
                    add_if_inside(gxb, a, q.y0 + 1, q.x0, c, gm * q.ly * (1.f - q.lx));
                    add_if_inside(gxb, a, q.y0 + 1, q.x0 + 1, c, gm * q.ly * q.lx);
                    s_dy += gm * ((1.f - q.lx) * (v10 - v00) + q.lx * (v11 - v01));
                    s_dx += gm * ((1.f - q.ly) * (v01 - v00) + q.ly * (v11 - v10));
                    s_m += gc * ((1.f - q.ly) * ((1.f - q.lx) * v00 + q.lx * v01) +
                                 q.ly * ((1.f - q.lx) * v10 + q.lx * v11));
                }
        }
    }
    if (goff == nullptr && gmask == nullptr) return;
    red[0][threadIdx.x] = s_dy;
    red[1][threadIdx.x] = s_dx;
    red[2][threadIdx.x] = s_m;
    __syncthreads();
    for (int st = blockDim.x / 2; st > 0; st >>= 1) {
        if ((int)threadIdx.x < st) {
            red[0][threadIdx.x] += red[0][threadIdx.x + st];
            red[1][threadIdx.x] += red[1][threadIdx.x + st];
            red[2][threadIdx.x] += red[2][threadIdx.x + st];
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        const bool live = g.b >= 0;
        if (goff) {
            goff[(size_t)r * 2 * kk + 2 * t] = live ? red[0][0] * a.gamma * g.h : 0.f;
            goff[(size_t)r * 2 * kk + 2 * t + 1] = live ? red[1][0] * a.gamma * g.w : 0.f;
        }
        if (gmask) gmask[(size_t)r * kk + t] = live ? red[2][0] : 0.f;
    }
}

// As droi_bwd_kernel, 16 bytes of channels per thread over the bin's pixel box
// (BinBox): grad_x gets each box pixel's share m/n * grad_y * wy * wx once, by
// 16-byte vector atomics; the offset gradients telescope over the sample rows
// (columns) to the box's last minus its first pixel row (column), and the mask
// gradient is the box sum. C a multiple of 16 bytes; x, grad_y and grad_x
// 16-byte aligned.
template <typename T>
__global__ void __launch_bounds__(256) droi_bwd_vec_kernel(RoiArgs a, const T* __restrict__ x,
                                                           const T* __restrict__ off, const T* __restrict__ mask,
                                                           const T* __restrict__ gy, float* __restrict__ gx,
                                                           float* __restrict__ goff, float* __restrict__ gmask) {
    constexpr int N = Vec16<T>::N;
    __shared__ float red[3][256];
    const int bin = blockIdx.x, kk = a.k * a.k;
    const int r = bin / kk, t = bin - r * kk;
    const BinGeom g = bin_geom(a, off, mask, r, t);
    float s_dy = 0.f, s_dx = 0.f, s_m = 0.f;
    const BinBox bx = bin_box(g);
    if (g.b >= 0 && bx.nu > 0 && bx.nv > 0) {
        const T* xb = x + (size_t)g.b * a.H * a.W * a.C;
        float* gxb = gx + (size_t)g.b * a.H * a.W * a.C;
        const T* gyb = gy + (size_t)bin * a.C;
        for (int cv = threadIdx.x; cv < a.C / N; cv += blockDim.x) {
            const int c = cv * N;
            float gc[N], gm[N], dyv[N], dxv[N], mv[N];
            load16(gyb + c, gc);
#pragma unroll
            for (int e = 0; e < N; ++e) {
                gc[e] /= g.n;
                gm[e] = gc[e] * g.m;
                dyv[e] = dxv[e] = mv[e] = 0.f;
            }
            for (int ra = 0; ra <= bx.nu; ++ra) {
                const int rr = bx.y0 + ra;
                if (rr < 0 || rr >= a.H) continue;
                const float wy = box_w(ra, bx.nu, bx.ly);
                const float sy = ra == bx.nu ? 1.f : (ra == 0 ? -1.f : 0.f);
                for (int cb = 0; cb <= bx.nv; ++cb) {
                    const int cc = bx.x0 + cb;
                    if (cc < 0 || cc >= a.W) continue;
                    const float wx = box_w(cb, bx.nv, bx.lx), wt = wy * wx;
                    const float sx = cb == bx.nv ? 1.f : (cb == 0 ? -1.f : 0.f);
                    const size_t o = ((size_t)rr * a.W + cc) * a.C + c;
                    float vv[N];
                    load16(xb + o, vv);
                    if (wt != 0.f)  // a box edge of zero weight (a fraction of exactly 0) adds nothing
#pragma unroll
                        for (int q = 0; q < N; q += 4)
                            ptx::red_add_v4(gxb + o + q, gm[q] * wt, gm[q + 1] * wt, gm[q + 2] * wt, gm[q + 3] * wt);
#pragma unroll
                    for (int e = 0; e < N; ++e) {
                        mv[e] += wt * vv[e];
                        dyv[e] += (sy * wx) * vv[e];
                        dxv[e] += (sx * wy) * vv[e];
                    }
                }
            }
#pragma unroll
            for (int e = 0; e < N; ++e) {
                s_dy += gm[e] * dyv[e];
                s_dx += gm[e] * dxv[e];
                s_m += gc[e] * mv[e];
            }
        }
    }
    if (goff == nullptr && gmask == nullptr) return;
    red[0][threadIdx.x] = s_dy;
    red[1][threadIdx.x] = s_dx;
    red[2][threadIdx.x] = s_m;
    __syncthreads();
    for (int st = blockDim.x / 2; st > 0; st >>= 1) {
        if ((int)threadIdx.x < st) {
            red[0][threadIdx.x] += red[0][threadIdx.x + st];
            red[1][threadIdx.x] += red[1][threadIdx.x + st];
            red[2][threadIdx.x] += red[2][threadIdx.x + st];
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        const bool live = g.b >= 0;
        if (goff) {
            goff[(size_t)r * 2 * kk + 2 * t] = live ? red[0][0] * a.gamma * g.h : 0.f;
            goff[(size_t)r * 2 * kk + 2 * t + 1] = live ? red[1][0] * a.gamma * g.w : 0.f;
        }
        if (gmask) gmask[(size_t)r * kk + t] = live ? red[2][0] : 0.f;
    }
}

// a power of two from 32 to 256 covering the channels (the reduction halves it)
int block_for(int C) {
    int t = 32;
    while (t < C && t < 256) t *= 2;
    return t;
}

}  // namespace

cudaError_t droi_forward(const RoiArgs& a, int dtype_bf16, const void* x, const void* off, const void* mask, void* y,
                         cudaStream_t st) {
    const long long bins = (long long)a.R * a.k * a.k;
    if (bins == 0) return cudaSuccess;
    const int es = dtype_bf16 ? 2 : 4, n = 16 / es;
    const bool vec = a.C % n == 0 && (reinterpret_cast<uintptr_t>(x) & 15) == 0 &&
                     (reinterpret_cast<uintptr_t>(y) & 15) == 0;
    if (vec && dtype_bf16)
        droi_fwd_vec_kernel<bf16><<<(unsigned)bins, block_for(a.C / n), 0, st>>>(
            a, (const bf16*)x, (const bf16*)off, (const bf16*)mask, (bf16*)y);
    else if (vec)
        droi_fwd_vec_kernel<float><<<(unsigned)bins, block_for(a.C / n), 0, st>>>(
            a, (const float*)x, (const float*)off, (const float*)mask, (float*)y);
    else if (dtype_bf16)
        droi_fwd_kernel<bf16><<<(unsigned)bins, block_for(a.C), 0, st>>>(a, (const bf16*)x, (const bf16*)off,
                                                                         (const bf16*)mask, (bf16*)y);
    else
        droi_fwd_kernel<float><<<(unsigned)bins, block_for(a.C), 0, st>>>(a, (const float*)x, (const float*)off,
                                                                          (const float*)mask, (float*)y);
    return cudaGetLastError();
}

cudaError_t droi_backward(const RoiArgs& a, int dtype_bf16, const void* x, const void* off, const void* mask,
                          const void* gy, float* gx, float* goff, float* gmask, cudaStream_t st) {
    const long long bins = (long long)a.R * a.k * a.k;
    if (bins == 0) return cudaSuccess;
    const int es = dtype_bf16 ? 2 : 4, n = 16 / es;
    const bool vec = a.C % n == 0 && (reinterpret_cast<uintptr_t>(x) & 15) == 0 &&
                     (reinterpret_cast<uintptr_t>(gy) & 15) == 0 && (reinterpret_cast<uintptr_t>(gx) & 15) == 0;
    if (vec && dtype_bf16)
        droi_bwd_vec_kernel<bf16><<<(unsigned)bins, block_for(a.C / n), 0, st>>>(
            a, (const bf16*)x, (const bf16*)off, (const bf16*)mask, (const bf16*)gy, gx, goff, gmask);
    else if (vec)
        droi_bwd_vec_kernel<float><<<(unsigned)bins, block_for(a.C / n), 0, st>>>(
            a, (const float*)x, (const float*)off, (const float*)mask, (const float*)gy, gx, goff, gmask);
    else if (dtype_bf16)
        droi_bwd_kernel<bf16><<<(unsigned)bins, block_for(a.C), 0, st>>>(
            a, (const bf16*)x, (const bf16*)off, (const bf16*)mask, (const bf16*)gy, gx, goff, gmask);
    else
        droi_bwd_kernel<float><<<(unsigned)bins, block_for(a.C), 0, st>>>(
            a, (const float*)x, (const float*)off, (const float*)mask, (const float*)gy, gx, goff, gmask);
    return cudaGetLastError();
}

}  // namespace dcn
