/*
 * dcn.h — C ABI of libdcn_b200, a CUDA library (sm_100a, NVIDIA B200) for the
 * modulated deformable convolution (DCNv2) with torchvision deform_conv2d
 * semantics.
 *
 * The operation ("Deformable ConvNets" notes, section "可变形卷积": the plain
 * convolution y(p0) = sum_{p_n in R} w(p_n) x(p0 + p_n) and its deformable form
 * with a learned offset dp_n per tap; DCNv2 section 3.2 adds a modulation
 * scalar m_k per tap):
 *
 *   y[b,ho,wo,o] = bias[o] + sum_{g<G} sum_{i,j<K} m * sum_{c in group g}
 *                  w[o,i,j,c] * bilinear(x[b,:,:,c], py, px)
 *   k  = i*K + j
 *   py = ho*stride - pad + i*dil + offset[b, g*2K^2 + 2k,     ho, wo]   (row,    "dy")
 *   px = wo*stride - pad + j*dil + offset[b, g*2K^2 + 2k + 1, ho, wo]   (column, "dx")
 *   m  = mask[b, g*K^2 + k, ho, wo]   (mask == NULL: m = 1, i.e. DCNv1)
 *
 * bilinear() weights the four integer neighbours of (py, px) by the areas of
 * the opposite sub-rectangles (notes, "双线性插值" S1..S4); a neighbour outside
 * [0,H) x [0,W) contributes zero (no clamping). Channels are split into G
 * deformable groups of Cin/G channels sharing one offset field (notes,
 * "Deformable Group"). Output size: Ho = (H + 2*pad - dil*(K-1) - 1)/stride + 1,
 * likewise Wo.
 *
 * Layouts (row-major, innermost dimension last; every tensor dense):
 *   x        [B, H, W, Cin]        channel-contiguous (NHWC)
 *   offset   [B, 2*G*K*K, Ho, Wo]
 *   mask     [B, G*K*K, Ho, Wo]
 *   weight   [Cout, K, K, Cin]     i.e. [Cout, K*K*Cin], tap-major then channel
 *   bias     [Cout]
 *   y        [B, Ho, Wo, Cout]
 *   grad_*   float32, laid out like the tensor they differentiate
 *
 * Element types: x, offset, mask, weight, bias, y and grad_y all have the type
 * given by dcn_params_t.dtype (DCN_F32: float, DCN_BF16: bfloat16). Gradients
 * are always float32. Arithmetic is float32 (coordinates, bilinear weights,
 * accumulation); on the bfloat16 path the modulated samples are rounded to
 * bfloat16 once, as tensor-core operands.
 *
 * Ownership and streams: every pointer except `params` is a DEVICE pointer
 * owned by the caller. The library never allocates device memory and never
 * synchronises: all work is enqueued on `stream` (a cudaStream_t; NULL is the
 * legacy default stream) of the current device, and returns as soon as it is
 * enqueued. Some calls need a caller-provided device workspace of
 * dcn_workspace_size() bytes (may be NULL when that size is 0). Outputs are
 * overwritten, never accumulated into.
 *
 * Errors: every entry point returns DCN_OK (0) or a negative code, and checks
 * its arguments before enqueueing anything. dcn_last_error_string() gives the
 * calling thread's last message. Device-side waits are bounded; a wait that
 * runs out records DCN_ERR_TIMEOUT in a device status word that
 * dcn_check_status() reads.
 */
#ifndef DCN_B200_H
#define DCN_B200_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DCN_ABI_VERSION 2

#if defined(__GNUC__)
#define DCN_API __attribute__((visibility("default")))
#else
#define DCN_API
#endif

typedef enum {
    DCN_F32 = 0,  /* float32 inputs and y */
    DCN_BF16 = 1  /* bfloat16 inputs and y */
} dcn_dtype_t;

/* Status codes. */
#define DCN_OK 0
#define DCN_ERR_INVALID_ARG (-1) /* a size is non-positive, Cin % G != 0, Ho or Wo <= 0, a required pointer is NULL */
#define DCN_ERR_UNSUPPORTED (-2) /* unknown dtype, pointer not aligned to its element size, size beyond int32 indexing */
#define DCN_ERR_CUDA (-3)        /* a CUDA call or launch failed; the message names it */
#define DCN_ERR_TIMEOUT (-4)     /* a bounded device wait ran out (reported by dcn_check_status) */
#define DCN_ERR_WORKSPACE (-5)   /* workspace NULL or smaller than dcn_workspace_size() */
#define DCN_ERR_RANGE (-6)       /* range-checked build only: a device access fell outside its buffer and was
                                    skipped (reported by dcn_check_status) */

/* dcn_params_t.flags */
#define DCN_FLAG_GENERIC 0x1u    /* use the generic CUDA-core kernels even where a specialised kernel exists */
#define DCN_FLAG_NO_TF32 0x2u    /* float32 layers: keep the contraction on CUDA cores (no split-tf32 tensor-core kernel) */

typedef struct dcn_params {
    int B, H, W;     /* batch, input height and width */
    int Cin, Cout;   /* input / output channels; Cin % G == 0 */
    int K;           /* square kernel size */
    int stride, pad, dil;
    int G;           /* deformable groups */
    int dtype;       /* dcn_dtype_t */
    unsigned flags;  /* DCN_FLAG_* */
} dcn_params_t;

/* Operation selectors for dcn_workspace_size(). */
#define DCN_OP_FORWARD 0
#define DCN_OP_BACKWARD_DATA 1   /* dcn_backward_data, dcn_backward_input, dcn_backward_offset_mask */
#define DCN_OP_BACKWARD_WEIGHT 2

/* Library ABI version (DCN_ABI_VERSION). */
DCN_API int dcn_abi_version(void);

/* Output size of the layer (the standard convolution formula above).
 * Returns DCN_ERR_INVALID_ARG when a size is invalid or Ho/Wo would be <= 0. */
DCN_API int dcn_output_size(const dcn_params_t* params, int* Ho, int* Wo);

/* Bytes of device workspace that the operation `op` (DCN_OP_*) needs for these
 * params; 0 when none. Returns 0 for invalid params as well (the call itself
 * then reports the error). */
DCN_API size_t dcn_workspace_size(const dcn_params_t* params, int op);

/* Forward pass: y = DCNv2(x, offset, mask, weight, bias).
 * mask and bias may be NULL. Writes y. */
DCN_API int dcn_forward(const dcn_params_t* params, const void* x, const void* offset, const void* mask,
                const void* weight, const void* bias, void* y, void* workspace, size_t workspace_bytes,
                void* stream);

/* Data-side backward in one pass: the gradients with respect to the input, the
 * offsets and the mask, given grad_y = dL/dy. Any of grad_x, grad_offset,
 * grad_mask may be NULL (not computed); grad_mask must be NULL when mask is
 * NULL. The offset gradient is taken through floor(): at an exact integer
 * sampling coordinate it is the right-hand derivative (the pages note the
 * bilinear kink there: the torchvision tutorial, section 3.2). */
DCN_API int dcn_backward_data(const dcn_params_t* params, const void* x, const void* offset, const void* mask,
                      const void* weight, const void* grad_y, float* grad_x, float* grad_offset, float* grad_mask,
                      void* workspace, size_t workspace_bytes, void* stream);

/* grad_x only (dcn_backward_data with grad_offset = grad_mask = NULL). */
DCN_API int dcn_backward_input(const dcn_params_t* params, const void* x, const void* offset, const void* mask,
                       const void* weight, const void* grad_y, float* grad_x, void* workspace,
                       size_t workspace_bytes, void* stream);

/* grad_offset and grad_mask (dcn_backward_data with grad_x = NULL). grad_mask may
 * be NULL; it must be NULL when mask is NULL. */
DCN_API int dcn_backward_offset_mask(const dcn_params_t* params, const void* x, const void* offset, const void* mask,
                             const void* weight, const void* grad_y, float* grad_offset, float* grad_mask,
                             void* workspace, size_t workspace_bytes, void* stream);

/* Weight-side backward: grad_weight [Cout, K, K, Cin] = sum over output pixels of
 * grad_y[p, o] * m * bilinear sample, and grad_bias [Cout] = sum_p grad_y[p, o]
 * (grad_bias may be NULL). */
DCN_API int dcn_backward_weight(const dcn_params_t* params, const void* x, const void* offset, const void* mask,
                        const void* grad_y, float* grad_weight, float* grad_bias, void* workspace,
                        size_t workspace_bytes, void* stream);

/* Forward pass that allocates nothing and takes no workspace. The pages have
 * no counterpart to this entry point; it exists for callers that cannot
 * allocate device memory themselves: code whose device memory is owned by
 * another allocator it cannot reach, and code that must not call cudaMalloc
 * during steady-state work because cudaMalloc can synchronize the device.
 *
 * Same arguments, layouts and results as dcn_forward, without workspace. Where
 * the forward needs scratch (the tensor-core path keeps float32 partial tiles,
 * per-tile counters, a reordered copy of the weights and the sampling records
 * there), it uses one static device array of
 * 48 MiB (50331648 bytes) compiled into the library; every GPU that loads the
 * library holds that array until the process exits. Shapes whose scratch
 * would exceed it are rejected with DCN_ERR_WORKSPACE and a message giving
 * both sizes, before anything is enqueued. The tile counters are cleared on
 * `stream` before each kernel runs. All calls on a device share the one
 * array, so calls whose work can overlap on the GPU (different streams, or
 * different host threads) race and may produce wrong results: issue them in
 * one stream order. The first call on each device looks up the array's
 * device address; make that first call before any stream capture. */
DCN_API int dcn_forward_noalloc(const dcn_params_t* params, const void* x, const void* offset, const void* mask,
                                const void* weight, const void* bias, void* y, void* stream);

/* Offset/mask predictor of a DCNv2 layer (notes, DCNv2 section 3.2, the
 * paragraph after the modulated y(p0) equation): a plain convolution over the
 * layer's input x with the layer's kernel size, stride, padding and dilation
 * and 3*G*K*K output channels. The first 2*G*K*K outputs are the offsets, the
 * remaining G*K*K pass through a sigmoid, 1 / (1 + exp(-v)), computed in
 * float32, and are the masks. params describes the DCN layer the outputs feed:
 * B, H, W, Cin, K, stride, pad, dil, G, dtype and flags are used, Cout is not.
 *   x       [B, H, W, Cin]                (as for dcn_forward)
 *   w_pred  [3*G*K*K, K, K, Cin]          (output channel, tap row, tap column, input channel)
 *   b_pred  [3*G*K*K], may be NULL (no bias)
 *   offset  [B, 2*G*K*K, Ho, Wo]          written; the layout dcn_forward reads
 *   mask    [B, G*K*K, Ho, Wo]            written
 * All in params->dtype, device memory owned by the caller, element-aligned.
 * bfloat16 layers of stride 1 with Cin a multiple of 8, 3*G*K*K <= 256 and
 * padded rows (W + 2*pad) short enough for the kernel's shared memory (up to
 * 212 pixels at K = 3) run one tensor-core kernel (float32
 * accumulation, the sigmoid in float32, outputs rounded to bfloat16 once): it
 * needs no workspace (dcn_predict_workspace_size returns 0 exactly when this
 * kernel applies) and 16-byte aligned x and w_pred (DCN_ERR_UNSUPPORTED
 * otherwise). Other layers run the convolution on this
 * library's forward kernels with zero offsets and no mask, one group and the
 * outputs padded to a multiple of 32, then split it; their precision is the
 * forward's for that shape, and they need workspace: device memory of at
 * least dcn_predict_workspace_size(params) bytes, 256-byte aligned, used as
 * scratch for the duration of the stream work.
 * Errors as for dcn_forward: argument problems return before anything is
 * enqueued; DCN_ERR_WORKSPACE when a needed workspace is NULL or too small. */
DCN_API size_t dcn_predict_workspace_size(const dcn_params_t* params);
DCN_API int dcn_predict_offset_mask(const dcn_params_t* params, const void* x, const void* w_pred,
                                    const void* b_pred, void* offset, void* mask, void* workspace,
                                    size_t workspace_bytes, void* stream);

/* (Modulated) deformable RoI pooling (notes, "可变形ROI pooling"; the explainer's
 * "可变形RoI池化" paragraph; DCNv2 section 3.2 for the per-bin modulation). The
 * pages describe it in words only; the computation is this reading of them:
 *   roi r = (b, x1, y1, x2, y2) in feature-map pixel coordinates, b truncated
 *   toward zero; h = max(y2 - y1, 0), w = max(x2 - x1, 0);
 *   bin t = i*k + j holds the integer offsets (u, v) with
 *     floor(i*h/k) <= u < ceil((i+1)*h/k),  floor(j*w/k) <= v < ceil((j+1)*w/k),
 *   n of them; its shift is (dy, dx) = gamma * (offset[r][2t] * h, offset[r][2t+1] * w);
 *   y[r][i][j][c] = m / n * sum over (u, v) of x_b(y1 + u + dy, x1 + v + dx, c),
 *   m = mask[r][t] (1 when mask is NULL), bilinear sampling whose neighbours
 *   outside the map contribute zero (as in the layer); 0 for an empty bin or a
 *   batch index outside [0, B).
 * Layouts: x [B, H, W, C]; rois [R, 5] float32; offset [R, 2*k*k] (normalised;
 * NULL: plain RoI pooling); mask [R, k*k] or NULL; y and grad_y [R, k, k, C].
 * x, offset, mask, y and grad_y are in `dtype`; gradients are float32. The
 * caller owns all device buffers; work is enqueued on `stream`; argument
 * problems return before anything is enqueued. */
typedef struct {
    int B, H, W, C;   /* feature map x [B, H, W, C] */
    int R, k;         /* RoIs (R >= 0) and bins per side (1 <= k <= 64) */
    float gamma;      /* scale of the normalised offsets */
    int dtype;        /* DCN_F32 or DCN_BF16 */
    unsigned flags;   /* reserved, 0 */
} dcn_roi_params_t;

/* Writes y. */
DCN_API int dcn_droi_pool_forward(const dcn_roi_params_t* params, const void* x, const float* rois,
                                  const void* offset, const void* mask, void* y, void* stream);

/* Given grad_y = dL/dy: grad_x (required, overwritten), grad_offset [R, 2*k*k]
 * (with respect to the normalised offsets; NULL: not computed; must be NULL
 * when offset is NULL) and grad_mask [R, k*k] (NULL: not computed; must be NULL
 * when mask is NULL). The RoI coordinates get no gradient. The offset gradient
 * is taken through floor(), as in the layer. grad_x is accumulated with float
 * atomics, so its last bits may differ between runs. */
DCN_API int dcn_droi_pool_backward(const dcn_roi_params_t* params, const void* x, const float* rois,
                                   const void* offset, const void* mask, const void* grad_y, float* grad_x,
                                   float* grad_offset, float* grad_mask, void* stream);

/* The calling thread's last error message ("" after success). */
DCN_API const char* dcn_last_error_string(void);

/* Waits for the work enqueued on `stream` so far (and for nothing else: other
 * streams keep running), then takes the device status word of the current
 * device, leaving it cleared, with one atomic exchange enqueued on `stream`.
 * The word collects the bounded-wait timeouts of every kernel of this library
 * on the device, whichever stream launched it; a kernel still running on
 * another stream may report after this call. Returns DCN_OK, or
 * DCN_ERR_TIMEOUT if a kernel gave up a bounded wait since the word was last
 * taken, or (range-checked build only, see DCN_ERR_RANGE) DCN_ERR_RANGE if a
 * checked device access fell outside its buffer and was skipped, or
 * DCN_ERR_CUDA if the stream reported an error. Enqueues one kernel (counted
 * by dcn_launch_count). */
DCN_API int dcn_check_status(void* stream);

/* Failure-detection self-test (no counterpart on the pages): enqueues one
 * kernel whose bounded mbarrier wait can never complete, through the same wait
 * every tensor-core kernel uses; after limit_cycles clock cycles (1e3 to 4e9)
 * it gives up, records the timeout in the device status word and ends
 * normally. The next dcn_check_status() returns DCN_ERR_TIMEOUT (and clears the
 * word); the context stays usable. Nothing faults, traps or hangs. */
DCN_API int dcn_selftest_wait_timeout(unsigned long long limit_cycles, void* stream);

/* Number of kernels (and memsets) this library has enqueued since the process
 * started, summed over threads. */
DCN_API unsigned long long dcn_launch_count(void);

/* Name of the kernel path the forward would take for these params (static
 * string), e.g. "tcgen05_gather" or "generic"; "invalid" for bad params. */
DCN_API const char* dcn_forward_path(const dcn_params_t* params);

#ifdef __cplusplus
}
#endif

#endif /* DCN_B200_H */
