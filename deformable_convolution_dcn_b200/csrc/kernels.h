// Internal launchers of libdcn_b200 (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include <atomic>

#include "common.cuh"

namespace dcn {

// generic.cu — CUDA-core kernels for every shape; dtype 0 = float, 1 = bfloat16.
cudaError_t generic_forward(const Shape& s, int dtype, const void* x, const void* off, const void* mask,
                            const void* w, const void* bias, void* y, cudaStream_t st);
cudaError_t generic_backward_data(const Shape& s, int dtype, const void* x, const void* off, const void* mask,
                                  const void* w, const void* gy, float* gx, float* goff, float* gmask,
                                  cudaStream_t st);
cudaError_t generic_backward_weight(const Shape& s, int dtype, const void* x, const void* off, const void* mask,
                                    const void* gy, float* gw, cudaStream_t st);
cudaError_t bias_grad(const Shape& s, int dtype, const void* gy, float* gb, cudaStream_t st, bool pdl = false);

// fwd_tc.cu — bfloat16 forward on tcgen05 tensor cores with the fused deformable gather.
bool fwd_tc_supported(const Shape& s);
size_t fwd_tc_workspace(const Shape& s);
cudaError_t fwd_tc(const Shape& s, const void* x, const void* off, const void* mask, const void* w, const void* bias,
                   void* y, void* ws, size_t ws_bytes, unsigned* status, cudaStream_t st, int* launches);

// fwd_tc_ts.cu — the same forward with the gathered operand in tensor memory (Cout <= 256);
// fwd_tc() dispatches to it where it applies.
bool fwd_ts_supported(const Shape& s);
size_t fwd_ts_workspace(const Shape& s);
cudaError_t fwd_ts(const Shape& s, const void* x, const void* off, const void* mask, const void* w, const void* bias,
                   void* y, void* ws, size_t ws_bytes, unsigned* status, cudaStream_t st, int* launches);
// Which of the two fwd_tc() runs for this shape ("tcgen05_gather_tmem" or "tcgen05_gather").
const char* fwd_tc_variant(const Shape& s);

// Same forward with its scratch in a static device array instead of a caller workspace.
size_t fwd_tc_static_scratch_bytes();
cudaError_t fwd_tc_noalloc(const Shape& s, const void* x, const void* off, const void* mask, const void* w,
                           const void* bias, void* y, unsigned* status, cudaStream_t st, int* launches);

// droi_pool.cu — (modulated) deformable RoI pooling, forward and backward (grad_x zeroed by the caller).
struct RoiArgs {
    const float* rois;  // [R, 5]: b, x1, y1, x2, y2
    int B, H, W, C, R, k;
    float gamma;
};
cudaError_t droi_forward(const RoiArgs& a, int dtype_bf16, const void* x, const void* off, const void* mask, void* y,
                         cudaStream_t st);
cudaError_t droi_backward(const RoiArgs& a, int dtype_bf16, const void* x, const void* off, const void* mask,
                          const void* gy, float* gx, float* goff, float* gmask, cudaStream_t st);

// pred_tc.cu — the bfloat16 stride-1 offset/mask predictor on tcgen05, sigmoid and split fused (no workspace).
bool pred_tc_supported(const Shape& s);
cudaError_t pred_tc(const Shape& s, const void* x, const void* w, const void* bias, void* off, void* mask,
                    unsigned* status, cudaStream_t st);

// predict.cu — the offset/mask predictor's weight padding and output split.
cudaError_t predict_pad(int dtype_bf16, const void* w, const void* b, void* wpad, void* bpad, int nc, int np, int kc,
                        cudaStream_t st);
cudaError_t predict_split(int dtype_bf16, const void* y, void* off, void* mask, int P, int plane, int np, int no,
                          int nc, cudaStream_t st);

// fwd_f32_tc.cu — float32 forward for layers with Cin <= 3, K*K <= 9 on tcgen05
// (split tf32 operands, float32 accuracy); y 16-byte aligned.
bool fwd_f32_tc_supported(const Shape& s);
cudaError_t fwd_f32_tc(const Shape& s, const void* x, const void* off, const void* mask, const void* w,
                       const void* bias, void* y, unsigned* status, cudaStream_t st);

// fwd_f32_stem.cu — the same float32 layers with Cout <= 128, one CTA per SM over an equal share
// of the output rows (a row-per-thread kernel for Cout 32 or 64, a persistent double-buffered one
// above); fwd_f32_tc() dispatches to it where it applies.
bool fwd_f32_stem_supported(const Shape& s);
cudaError_t fwd_f32_stem(const Shape& s, const void* x, const void* off, const void* mask, const void* w,
                         const void* bias, void* y, unsigned* status, cudaStream_t st);

// fwd_f32_small.cu — float32 forward for layers with Cin <= 8 (CUDA cores, HBM-bound).
bool fwd_f32_small_supported(const Shape& s);
cudaError_t fwd_f32_small(const Shape& s, const void* x, const void* off, const void* mask, const void* w,
                          const void* bias, void* y, cudaStream_t st);

// fwd_tc_ts.cu, transposed pass — grad_x of a bfloat16 layer (channels per group
// <= 256) as a gather-GEMM on tcgen05, written outright (no atomics, no zeroing).
// Sample corners past a list's capacity are not included: they are flagged in
// ovf[(g*K2 + tap) * ovf_pitch + p] (bit n = corner n) for the caller to add.
// rec (optional): the float32 sampling records of bwd_data_tc.cu, written at
// the same index.
bool gxt_supported(const Shape& s);
size_t gxt_workspace(const Shape& s);
// zeroes the lists' counts and the flags; enqueue it before the kernel that gxt's
// first kernel follows (gxt launches it as that kernel's programmatic dependent)
cudaError_t gxt_prepare(const Shape& s, uint8_t* ovf, int ovf_pitch, void* ws, size_t ws_bytes, cudaStream_t st,
                        int* launches);
cudaError_t gxt(const Shape& s, const void* off, const void* mask, const void* w, const void* gy, float* gx,
                uint8_t* ovf, void* rec, int ovf_pitch, void* ws, size_t ws_bytes, unsigned* status,
                cudaStream_t st, int* launches);

// bwd_weight_tc.cu — bfloat16 weight gradient on tcgen05 (workspace: sampling records).
bool bwd_weight_tc_supported(const Shape& s);
size_t bwd_weight_tc_workspace(const Shape& s);
cudaError_t bwd_weight_tc(const Shape& s, const void* x, const void* off, const void* mask, const void* gy,
                          float* gw, void* ws, size_t ws_bytes, unsigned* status, cudaStream_t st, int* launches);

// bwd_data_tc.cu — bfloat16 grad_x / grad_offset / grad_mask on tcgen05 (workspace: records, w^T).
bool bwd_data_tc_supported(const Shape& s);
size_t bwd_data_tc_workspace(const Shape& s);
cudaError_t bwd_data_tc(const Shape& s, const void* x, const void* off, const void* mask, const void* w,
                        const void* gy, float* gx, float* goff, float* gmask, void* ws, size_t ws_bytes,
                        unsigned* status, cudaStream_t st, int* launches);

// bwd_gx_tc.cu — grad_x alone on tcgen05 with the scatter summed in a shared-memory window
// (groups of whole 32-channel slices); uses the data-backward pre-pass's records and W^T.
bool bwd_gx_supported(const Shape& s);
cudaError_t bwd_gx_tc(const Shape& s, const void* gy, const void* wt, const void* rec, int ppad, float* gx,
                      unsigned* status, cudaStream_t st, int* launches);

// selftest.cu — a kernel whose bounded wait can only give up (failure-detection test).
cudaError_t selftest_wait_timeout(long long limit_cycles, cudaStream_t st);

// status.cu — the device status word that bounded waits report to; SM count.
int num_sms();
cudaError_t status_word_ptr(unsigned int** ptr);
// Waits for `st`, then atomically takes the status word (leaving 0) and returns it in *out.
cudaError_t read_and_clear_status(unsigned int* out, cudaStream_t st);

// Per-device "done" flags for one-time host set-up (one per kernel), safe to
// test and set from several host threads at once.
struct DeviceFlags {
    std::atomic<bool> done[64];
};
// cudaFuncSetAttribute(func, MaxDynamicSharedMemorySize, bytes) once per device
// for the current device; later calls return at once. Thread-safe.
cudaError_t max_dynamic_smem_once(const void* func, int bytes, DeviceFlags& flags);
// Per-device cache of the last shared-memory carveout set for one kernel.
struct DeviceCarveout {
    std::atomic<int> pct[64];  // 0: not set yet, else percentage + 1
};
// Asks for the smallest shared-memory carveout that holds `smem_bytes` of
// dynamic shared memory for `func` on the current device, leaving the rest of
// the SM's unified L1 / shared memory to the L1 cache (re-set only when the
// needed percentage changes). Thread-safe.
cudaError_t smem_carveout_for(const void* func, uint32_t smem_bytes, DeviceCarveout& cache);

}  // namespace dcn
