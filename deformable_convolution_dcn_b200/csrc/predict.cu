// The offsets and modulation masks of a DCNv2 layer come from a separate plain
// convolution over the same input, at the layer's spatial resolution, with
// 3*G*K*K output channels: the first 2*G*K*K are the offsets, the rest pass
// through a sigmoid and become the masks (notes, DCNv2 section 3.2, the
// paragraph after the modulated y(p0) equation).
//
// A plain convolution is this library's layer with zero offsets and no mask
// (every sample falls on its top-left neighbour with weight 1), so the
// predictor runs the forward kernels on an all-zero offset tensor; the helpers
// here pad the predictor's weights to a multiple of 32 outputs and scatter the
// [P x NP] result (NHWC) into the offset and mask tensors ([B, C, Ho, Wo]),
// applying the sigmoid to the mask channels in float32.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace dcn {
namespace {

template <typename T>
__global__ void __launch_bounds__(256) pred_pad_kernel(const T* __restrict__ w, const T* __restrict__ b, T* __restrict__ wpad,
                                                      T* __restrict__ bpad, int nc, int np, int kc) {
    const long long n = (long long)np * kc;
    for (long long i = blockIdx.x * 256LL + threadIdx.x; i < n; i += (long long)gridDim.x * 256) {
        const int o = (int)(i / kc);
        wpad[i] = o < nc ? w[i] : from_float<T>(0.f);
    }
    if (blockIdx.x == 0)
        for (int o = threadIdx.x; o < np; o += 256) bpad[o] = (b != nullptr && o < nc) ? b[o] : from_float<T>(0.f);
}

// out channel ch of pixel p (raster order) -> offset[b][ch][pix] (ch < no) or
// mask[b][ch - no][pix] = sigmoid(value) (no <= ch < nc)
template <typename T>
__global__ void __launch_bounds__(256) pred_split_kernel(const T* __restrict__ y, T* __restrict__ off, T* __restrict__ mask,
                                                        int P, int plane, int np, int no, int nc) {
    const long long n = (long long)nc * P;
    for (long long i = blockIdx.x * 256LL + threadIdx.x; i < n; i += (long long)gridDim.x * 256) {
        const int ch = (int)(i / P), p = (int)(i - (long long)ch * P);  // consecutive threads: consecutive pixels
        const int b = p / plane, pix = p - b * plane;
        const float v = ldf(y + (size_t)p * np + ch);
        if (ch < no) {
            off[((size_t)b * no + ch) * plane + pix] = from_float<T>(v);
        } else {
            const int nm = nc - no;
            mask[((size_t)b * nm + (ch - no)) * plane + pix] = from_float<T>(1.f / (1.f + expf(-v)));
        }
    }
}

int grid_for(long long n) { return (int)std::min<long long>((n + 255) / 256, 4 * 148 * 8); }

}  // namespace

cudaError_t predict_pad(int dtype_bf16, const void* w, const void* b, void* wpad, void* bpad, int nc, int np, int kc,
                        cudaStream_t st) {
    const int g = grid_for((long long)np * kc);
    if (dtype_bf16)
        pred_pad_kernel<bf16><<<g, 256, 0, st>>>((const bf16*)w, (const bf16*)b, (bf16*)wpad, (bf16*)bpad, nc, np, kc);
    else
        pred_pad_kernel<float><<<g, 256, 0, st>>>((const float*)w, (const float*)b, (float*)wpad, (float*)bpad, nc, np,
                                                  kc);
    return cudaGetLastError();
}

cudaError_t predict_split(int dtype_bf16, const void* y, void* off, void* mask, int P, int plane, int np, int no,
                          int nc, cudaStream_t st) {
    const int g = grid_for((long long)nc * P);
    if (dtype_bf16)
        pred_split_kernel<bf16><<<g, 256, 0, st>>>((const bf16*)y, (bf16*)off, (bf16*)mask, P, plane, np, no, nc);
    else
        pred_split_kernel<float><<<g, 256, 0, st>>>((const float*)y, (float*)off, (float*)mask, P, plane, np, no, nc);
    return cudaGetLastError();
}

}  // namespace dcn
