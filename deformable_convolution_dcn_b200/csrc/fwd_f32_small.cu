// Forward DCNv2 in float32 for layers with few input channels (Cin <= 8), such
// as a 224x224 RGB stem layer (3 -> 64 channels). The contraction is only
// K*K*Cin deep (27 for the stem), too thin for tensor cores, and float32
// accuracy is required, so this is a CUDA-core kernel organised for HBM and
// latency:
//
//   phase 1  all 256 threads of a block build the block's column tile
//            col[pixel][tap*Cin + c] = m * bilinear(x, sample) in shared memory;
//            each thread takes up to five (pixel, tap) pairs and has all their
//            offset/mask loads, then all their neighbour loads, in flight at once;
//   phase 2  each thread contracts 4 pixels x 8 output channels against the
//            weights [K*K*Cin][Cout] held in shared memory;
//   phase 3  8 consecutive lanes store one pixel's output row contiguously.
#include "common.cuh"
#include "kernels.h"

namespace dcn {
namespace {

constexpr int THREADS = 256;
constexpr int PX_PER_THREAD = 4;     // phase 2 register block: 4 pixels
constexpr int OG = 8;                // ... x 8 output channels

// d += a * b on packed float pairs (two independent float32 FMAs, round to nearest).
__device__ __forceinline__ void fma2(unsigned long long& d, unsigned long long a, unsigned long long b) {
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(d) : "l"(a), "l"(b));
}

template <int CIN>
__global__ void __launch_bounds__(THREADS, 3) stem_fwd_kernel(Shape s, const float* __restrict__ x,
                                                           const float* __restrict__ off,
                                                           const float* __restrict__ mask,
                                                           const float* __restrict__ w,
                                                           const float* __restrict__ bias, float* __restrict__ y,
                                                           int px_per_block) {
    // (pixel, tap) pairs per thread per batch in phase 1, sized to the register budget
    constexpr int PAIRS_PER_THREAD = CIN <= 3 ? 3 : (CIN <= 5 ? 2 : 1);
    extern __shared__ float smem[];
    const int KC = s.K2 * CIN;       // contraction depth
    const int ldc = KC | 1;          // odd column-tile pitch: lanes on consecutive pixels hit distinct banks
    float* ws = smem;                // [KC][Cout]
    float* col = smem + KC * s.Cout; // [px_per_block][ldc]
    // per pixel: mask index of channel 0 (b*G*K2*plane + pix, -1 past the end), x image base, sampling origin
    int4* s_px = reinterpret_cast<int4*>(col + px_per_block * ldc);
    int* s_pix = reinterpret_cast<int*>(s_px + px_per_block);        // per pixel: in-plane index
    int2* s_tp = reinterpret_cast<int2*>(s_pix + px_per_block);      // per tap: (i*dil, j*dil)
    const int tid = threadIdx.x;
    // weights, transposed into [K*K*Cin][Cout]: every load of a batch is issued
    // before any is stored, and the batch's latency overlaps the tables below
    const int nw = KC * s.Cout;
    constexpr int WB = 8;
    float wr[WB];
#pragma unroll
    for (int q = 0; q < WB; ++q) {
        const int e = tid + q * THREADS;
        wr[q] = e < nw ? __ldg(w + e) : 0.f;
    }
    const int p0 = blockIdx.x * px_per_block;
    const int plane = s.Ho * s.Wo;
    const int npairs = px_per_block * s.K2 * s.G;
    const int lg = 31 - __clz(px_per_block);  // px_per_block is a power of two
    for (int px = tid; px < px_per_block; px += THREADS) {
        const int p = p0 + px;
        int4 r = make_int4(-1, 0, 0, 0);
        if (p < s.P) {
            const int b = p / plane, pix = p - b * plane;
            const int ho = pix / s.Wo, wo = pix - ho * s.Wo;
            r = make_int4(b * s.G * s.K2 * plane + pix, b * s.H * s.W * s.Cin, ho * s.stride - s.pad,
                          wo * s.stride - s.pad);
            s_pix[px] = pix;
        }
        s_px[px] = r;
    }
    for (int t = tid; t < s.K2; t += THREADS) {
        const int i = t / s.K;
        s_tp[t] = make_int2(i * s.dil, (t - i * s.K) * s.dil);
    }
    for (int e0 = 0; e0 < nw; e0 += WB * THREADS) {
        if (e0 > 0) {
#pragma unroll
            for (int q = 0; q < WB; ++q) {
                const int e = e0 + tid + q * THREADS;
                wr[q] = e < nw ? __ldg(w + e) : 0.f;
            }
        }
#pragma unroll
        for (int q = 0; q < WB; ++q) {
            const int e = e0 + tid + q * THREADS;  // stored order [Cout][K*K*Cin]
            if (e < nw) {
                const int o = e / KC, r = e - o * KC;
                ws[r * s.Cout + o] = wr[q];
            }
        }
    }
    __syncthreads();

    // ---------------------------------------------------------------- phase 1
    for (int e0 = 0; e0 < npairs; e0 += PAIRS_PER_THREAD * THREADS) {
        float dy[PAIRS_PER_THREAD], dx[PAIRS_PER_THREAD], mk[PAIRS_PER_THREAD];
        int pr[PAIRS_PER_THREAD];
#pragma unroll
        for (int q = 0; q < PAIRS_PER_THREAD; ++q) {
            const int e = e0 + q * THREADS + tid;
            const int gt = e >> lg, px = e & (px_per_block - 1);  // gt = g*K2 + tap
            pr[q] = (e < npairs) ? s_px[px].x : -1;
            dy[q] = dx[q] = 0.f;
            mk[q] = 0.f;
            if (pr[q] >= 0) {
                // with mb = b*GK2*plane + pix: mask index (b*GK2 + gt)*plane + pix = mb + gt*plane,
                // offset index (b*2GK2 + 2gt)*plane + pix = 2*mb - pix + 2*gt*plane
                const size_t mi = (size_t)pr[q] + (size_t)gt * plane;
                const size_t ob = 2 * (size_t)pr[q] - s_pix[px] + (size_t)2 * gt * plane;
                dy[q] = __ldg(off + ob);
                dx[q] = __ldg(off + ob + plane);
                mk[q] = mask ? __ldg(mask + mi) : 1.f;
            }
        }
        float v[PAIRS_PER_THREAD][4][CIN];
        float wt[PAIRS_PER_THREAD][4];
#pragma unroll
        for (int q = 0; q < PAIRS_PER_THREAD; ++q) {
            const int e = e0 + q * THREADS + tid;
            const int gt = e >> lg, px = e & (px_per_block - 1);
            const int g = (s.G == 1) ? 0 : gt / s.K2, tap = gt - g * s.K2;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                wt[q][k] = 0.f;
#pragma unroll
                for (int c = 0; c < CIN; ++c) v[q][k][c] = 0.f;
            }
            if (pr[q] < 0) continue;
            const int4 pi = s_px[px];
            const int2 to = s_tp[tap];
            int y0, x0;
            float ly, lx;
            split_coord(pi.z + to.x, dy[q], y0, ly);
            split_coord(pi.w + to.y, dx[q], x0, lx);
            const float* xb = x + (size_t)pi.y + g * s.Cg;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int r = y0 + (k >> 1), qq = x0 + (k & 1);
                if (!inside(s, r, qq)) continue;
                wt[q][k] = ((k >> 1) ? ly : 1.f - ly) * ((k & 1) ? lx : 1.f - lx) * mk[q];
                const float* pc = xb + ((size_t)r * s.W + qq) * s.Cin;
#pragma unroll
                for (int c = 0; c < CIN; ++c)
                    if (c < s.Cg) v[q][k][c] = __ldg(pc + c);
            }
        }
#pragma unroll
        for (int q = 0; q < PAIRS_PER_THREAD; ++q) {
            const int e = e0 + q * THREADS + tid;
            if (e >= npairs) continue;
            const int gt = e >> lg, px = e & (px_per_block - 1);
            const int g = (s.G == 1) ? 0 : gt / s.K2, tap = gt - g * s.K2;
#pragma unroll
            for (int c = 0; c < CIN; ++c) {
                if (c >= s.Cg) break;
                const float t = wt[q][0] * v[q][0][c] + wt[q][1] * v[q][1][c] + wt[q][2] * v[q][2][c] +
                                wt[q][3] * v[q][3][c];
                col[px * ldc + tap * CIN + g * s.Cg + c] = t;
            }
        }
    }
    __syncthreads();

    // ---------------------------------------------------------------- phase 2
    const int ogroups = s.Cout / OG;
    const int to = tid % ogroups, tp = tid / ogroups;  // output group, pixel group
    // accumulators as float pairs: acc2[u][h] holds output channels 2h, 2h+1 of pixel u
    unsigned long long acc2[PX_PER_THREAD][OG / 2];
#pragma unroll
    for (int u = 0; u < PX_PER_THREAD; ++u)
#pragma unroll
        for (int h = 0; h < OG / 2; ++h) acc2[u][h] = 0ull;
    const float* colr = col + (tp * PX_PER_THREAD) * ldc;
    for (int k = 0; k < KC; ++k) {
        const ulonglong2 wa = *reinterpret_cast<const ulonglong2*>(ws + k * s.Cout + to * OG);
        const ulonglong2 wb = *reinterpret_cast<const ulonglong2*>(ws + k * s.Cout + to * OG + 4);
#pragma unroll
        for (int u = 0; u < PX_PER_THREAD; ++u) {
            const float a = colr[u * ldc + k];
            const unsigned long long aa =
                ((unsigned long long)__float_as_uint(a) << 32) | (unsigned long long)__float_as_uint(a);
            fma2(acc2[u][0], aa, wa.x);
            fma2(acc2[u][1], aa, wa.y);
            fma2(acc2[u][2], aa, wb.x);
            fma2(acc2[u][3], aa, wb.y);
        }
    }
    float acc[PX_PER_THREAD][OG];
#pragma unroll
    for (int u = 0; u < PX_PER_THREAD; ++u)
#pragma unroll
        for (int h = 0; h < OG / 2; ++h) {
            acc[u][2 * h] = __uint_as_float((unsigned)(acc2[u][h] & 0xFFFFFFFFull));
            acc[u][2 * h + 1] = __uint_as_float((unsigned)(acc2[u][h] >> 32));
        }

    // ---------------------------------------------------------------- phase 3
    float bv[OG];
#pragma unroll
    for (int o = 0; o < OG; ++o) bv[o] = bias ? __ldg(bias + to * OG + o) : 0.f;
#pragma unroll
    for (int u = 0; u < PX_PER_THREAD; ++u) {
        const int p = p0 + tp * PX_PER_THREAD + u;
        if (p >= s.P) continue;
        float4* dst = reinterpret_cast<float4*>(y + (size_t)p * s.Cout + to * OG);
        dst[0] = make_float4(acc[u][0] + bv[0], acc[u][1] + bv[1], acc[u][2] + bv[2], acc[u][3] + bv[3]);
        dst[1] = make_float4(acc[u][4] + bv[4], acc[u][5] + bv[5], acc[u][6] + bv[6], acc[u][7] + bv[7]);
    }
}

size_t smem_bytes(const Shape& s, int cin, int px_per_block) {
    const int KC = s.K2 * cin;
    return ((size_t)KC * s.Cout + (size_t)px_per_block * (KC | 1)) * sizeof(float) + (size_t)px_per_block * 16 + 16 +
           (size_t)px_per_block * 4 + (size_t)s.K2 * 8 + 16;
}

int px_per_block(const Shape& s) { return (THREADS / (s.Cout / OG)) * PX_PER_THREAD; }

template <int CIN>
cudaError_t launch(const Shape& s, const float* x, const float* off, const float* mask, const float* w,
                   const float* bias, float* y, cudaStream_t st) {
    const int ppb = px_per_block(s);
    const size_t smem = smem_bytes(s, CIN, ppb);
    static DeviceFlags attr;
    cudaError_t e = cudaSuccess;
    if (smem > 48 * 1024) {
        e = max_dynamic_smem_once((const void*)stem_fwd_kernel<CIN>, 200 * 1024, attr);
        if (e != cudaSuccess) return e;
    }
    dim3 grid((s.P + ppb - 1) / ppb);
    stem_fwd_kernel<CIN><<<grid, THREADS, smem, st>>>(s, x, off, mask, w, bias, y, ppb);
    return cudaGetLastError();
}

}  // namespace

// Cin <= 8, Cout in {8, 16, 32, 64, 128, 256}, shared memory within 200 KB.
bool fwd_f32_small_supported(const Shape& s) {
    // Cout / 8 output groups must divide the 256 threads (so pixels per block is a power of two)
    if (s.Cin > 8 || s.Cout % OG || s.Cout < OG || s.Cout > THREADS || THREADS % (s.Cout / OG)) return false;
    return smem_bytes(s, s.Cin, px_per_block(s)) <= 200 * 1024 &&
           (long long)s.B * 2 * s.G * s.K2 * s.Ho * s.Wo < (1LL << 31) && (long long)s.B * s.H * s.W * s.Cin < (1LL << 31);
}

cudaError_t fwd_f32_small(const Shape& s, const void* x, const void* off, const void* mask, const void* w,
                          const void* bias, void* y, cudaStream_t st) {
    const float *xf = (const float*)x, *of = (const float*)off, *mf = (const float*)mask, *wf = (const float*)w,
                *bf = (const float*)bias;
    float* yf = (float*)y;
    switch (s.Cin) {
        case 1: return launch<1>(s, xf, of, mf, wf, bf, yf, st);
        case 2: return launch<2>(s, xf, of, mf, wf, bf, yf, st);
        case 3: return launch<3>(s, xf, of, mf, wf, bf, yf, st);
        case 4: return launch<4>(s, xf, of, mf, wf, bf, yf, st);
        case 5: return launch<5>(s, xf, of, mf, wf, bf, yf, st);
        case 6: return launch<6>(s, xf, of, mf, wf, bf, yf, st);
        case 7: return launch<7>(s, xf, of, mf, wf, bf, yf, st);
        default: return launch<8>(s, xf, of, mf, wf, bf, yf, st);
    }
}

}  // namespace dcn
