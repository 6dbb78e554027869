// Shared device helpers of libdcn_b200: the kernel-side shape, element loads,
// and the per-(pixel, tap, group) sampling arithmetic.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dcn {

// Layer geometry as the kernels see it (filled in by the host from dcn_params_t).
struct Shape {
    int B, H, W, Cin, Cout, K, stride, pad, dil, G;
    int Ho, Wo, K2, Cg;
    int P;       // output pixels B*Ho*Wo (the GEMM M)
    int KC;      // K*K*Cin (the GEMM K; row length of the weight)
};

typedef __nv_bfloat16 bf16;

template <typename T>
__device__ __forceinline__ float ldf(const T* p);
template <>
__device__ __forceinline__ float ldf<float>(const float* p) {
    return __ldg(p);
}
template <>
__device__ __forceinline__ float ldf<bf16>(const bf16* p) {
    return __bfloat162float(__ldg(p));
}

template <typename T>
__device__ __forceinline__ T from_float(float v);
template <>
__device__ __forceinline__ float from_float<float>(float v) {
    return v;
}
template <>
__device__ __forceinline__ bf16 from_float<bf16>(float v) {
    return __float2bfloat16_rn(v);
}

// Integer and fractional parts of the sampling coordinate base + d, where base
// is an integer: floor(base + d) = base + floor(d) exactly, and d - floor(d) is
// exact in float for the offsets' range, so the neighbour choice matches a
// float64 evaluation of floor(base + d). The floor is clamped to +-2^20 so that
// huge or non-finite offsets land far outside the map instead of overflowing.
__device__ __forceinline__ void split_coord(int base, float d, int& i0, float& frac) {
    float fl = floorf(d);
    fl = fminf(fmaxf(fl, -1048576.f), 1048576.f);
    i0 = base + (int)fl;
    frac = d - floorf(d);
    if (!(frac >= 0.f && frac <= 1.f)) frac = 0.f;  // non-finite offset: the sample is outside anyway
}

// Sampling of tap k = i*K + j of group g at output pixel p = (b, ho, wo).
struct TapSample {
    int b, y0, x0;   // top-left neighbour (may lie outside the map)
    float ly, lx;    // fractional parts
    float m;         // modulation scalar
};

template <typename T>
__device__ __forceinline__ TapSample tap_sample(const Shape& s, const T* off, const T* mask, int p, int g, int tap) {
    TapSample t;
    int plane = s.Ho * s.Wo;
    t.b = p / plane;
    int pix = p - t.b * plane;
    int ho = pix / s.Wo, wo = pix - (pix / s.Wo) * s.Wo;
    int i = tap / s.K, j = tap - (tap / s.K) * s.K;
    size_t ob = ((size_t)t.b * 2 * s.G * s.K2 + (size_t)g * 2 * s.K2 + 2 * tap) * plane + pix;
    float dy = ldf(off + ob);
    float dx = ldf(off + ob + plane);
    t.m = mask ? ldf(mask + ((size_t)t.b * s.G * s.K2 + (size_t)g * s.K2 + tap) * plane + pix) : 1.f;
    split_coord(ho * s.stride - s.pad + i * s.dil, dy, t.y0, t.ly);
    split_coord(wo * s.stride - s.pad + j * s.dil, dx, t.x0, t.lx);
    return t;
}

__device__ __forceinline__ bool inside(const Shape& s, int r, int q) {
    return (unsigned)r < (unsigned)s.H && (unsigned)q < (unsigned)s.W;
}

// Bilinear sample of channel c (no modulation); zero for neighbours outside.
template <typename T>
__device__ __forceinline__ float bilinear_at(const Shape& s, const T* x, const TapSample& t, int c) {
    const T* xb = x + (size_t)t.b * s.H * s.W * s.Cin + c;
    float v = 0.f;
    if (inside(s, t.y0, t.x0)) v += (1.f - t.ly) * (1.f - t.lx) * ldf(xb + ((size_t)t.y0 * s.W + t.x0) * s.Cin);
    if (inside(s, t.y0, t.x0 + 1)) v += (1.f - t.ly) * t.lx * ldf(xb + ((size_t)t.y0 * s.W + t.x0 + 1) * s.Cin);
    if (inside(s, t.y0 + 1, t.x0)) v += t.ly * (1.f - t.lx) * ldf(xb + ((size_t)(t.y0 + 1) * s.W + t.x0) * s.Cin);
    if (inside(s, t.y0 + 1, t.x0 + 1)) v += t.ly * t.lx * ldf(xb + ((size_t)(t.y0 + 1) * s.W + t.x0 + 1) * s.Cin);
    return v;
}

}  // namespace dcn
