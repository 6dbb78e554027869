// C ABI of libdcn_b200 (declared in include/dcn.h): argument checks, workspace
// sizing and dispatch to the kernels. Nothing here computes the convolution;
// every step runs in the CUDA kernels.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <string>

#include "dcn.h"
#include "kernels.h"

// Built with -DDCN_NVTX, every entry point that enqueues device work opens an
// NVTX range named after itself for the duration of the call (host side: the
// enqueue, not the kernels), so that a timeline tool shows which library call
// launched which kernels. Header-only; no effect in the default build.
#ifdef DCN_NVTX
#include <nvtx3/nvToolsExt.h>
namespace {
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};
}  // namespace
#define DCN_TRACE(name) NvtxRange dcn_nvtx_range_(name)
#else
#define DCN_TRACE(name) ((void)0)
#endif

namespace {

thread_local std::string g_err;
std::atomic<unsigned long long> g_launches{0};

int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

int ok() {
    g_err.clear();
    return DCN_OK;
}

int cuda_fail(cudaError_t e, const char* what) {
    return fail(DCN_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
}

const long long kMaxElems = (1LL << 31) - 1;

// Validates params and fills the kernel-side shape. Returns DCN_OK or an error code (message set).
int make_shape(const dcn_params_t* p, dcn::Shape& s) {
    if (!p) return fail(DCN_ERR_INVALID_ARG, "params is NULL");
    if (p->B < 1 || p->H < 1 || p->W < 1 || p->Cin < 1 || p->Cout < 1 || p->K < 1 || p->stride < 1 || p->dil < 1 ||
        p->G < 1 || p->pad < 0)
        return fail(DCN_ERR_INVALID_ARG,
                    "sizes must be positive (B=%d H=%d W=%d Cin=%d Cout=%d K=%d stride=%d dil=%d G=%d) and pad >= 0 "
                    "(pad=%d)",
                    p->B, p->H, p->W, p->Cin, p->Cout, p->K, p->stride, p->dil, p->G, p->pad);
    if (p->Cin % p->G) return fail(DCN_ERR_INVALID_ARG, "Cin=%d is not a multiple of G=%d", p->Cin, p->G);
    if (p->dtype != DCN_F32 && p->dtype != DCN_BF16) return fail(DCN_ERR_UNSUPPORTED, "unknown dtype %d", p->dtype);
    if (p->H > (1 << 19) || p->W > (1 << 19) || p->K > 64 || p->pad > (1 << 19) || p->dil > (1 << 16) ||
        p->stride > (1 << 16))
        return fail(DCN_ERR_UNSUPPORTED, "H, W, pad up to 2^19, K up to 64, stride and dil up to 2^16");
    long long Ho = ((long long)p->H + 2LL * p->pad - (long long)p->dil * (p->K - 1) - 1) / p->stride + 1;
    long long Wo = ((long long)p->W + 2LL * p->pad - (long long)p->dil * (p->K - 1) - 1) / p->stride + 1;
    if ((long long)p->H + 2LL * p->pad - (long long)p->dil * (p->K - 1) - 1 < 0 ||
        (long long)p->W + 2LL * p->pad - (long long)p->dil * (p->K - 1) - 1 < 0 || Ho < 1 || Wo < 1)
        return fail(DCN_ERR_INVALID_ARG, "output would be empty: the dilated kernel does not fit the padded input");
    long long K2 = (long long)p->K * p->K;
    long long P = (long long)p->B * Ho * Wo;
    long long nx = (long long)p->B * p->H * p->W * p->Cin;
    long long noff = P * 2 * p->G * K2;
    long long ny = P * p->Cout;
    long long nw = (long long)p->Cout * K2 * p->Cin;
    if (nx > kMaxElems || noff > kMaxElems || ny > kMaxElems || nw > kMaxElems)
        return fail(DCN_ERR_UNSUPPORTED, "a tensor exceeds 2^31-1 elements");
    s.B = p->B;
    s.H = p->H;
    s.W = p->W;
    s.Cin = p->Cin;
    s.Cout = p->Cout;
    s.K = p->K;
    s.stride = p->stride;
    s.pad = p->pad;
    s.dil = p->dil;
    s.G = p->G;
    s.Ho = (int)Ho;
    s.Wo = (int)Wo;
    s.K2 = (int)K2;
    s.Cg = p->Cin / p->G;
    s.P = (int)P;
    s.KC = (int)(K2 * p->Cin);
    return DCN_OK;
}

size_t elem_size(int dtype) { return dtype == DCN_F32 ? 4 : 2; }

int check_ptr(const void* ptr, const char* name, size_t align, bool required) {
    if (!ptr) return required ? fail(DCN_ERR_INVALID_ARG, "%s is NULL", name) : DCN_OK;
    if ((uintptr_t)ptr % align)
        return fail(DCN_ERR_UNSUPPORTED, "%s is not aligned to %zu bytes", name, align);
    return DCN_OK;
}

bool aligned16(const void* p) { return p == nullptr || ((uintptr_t)p & 15) == 0; }

// The tensor-core forward takes bfloat16 layers whose channel counts are
// multiples of 8 (16-byte vectors) and at most 25 taps; pointers are checked
// separately at the call.
bool use_fwd_tc(const dcn_params_t* p, const dcn::Shape& s) {
    return p->dtype == DCN_BF16 && !(p->flags & DCN_FLAG_GENERIC) && dcn::fwd_tc_supported(s);
}

// The float32 tensor-core forward for RGB-like layers: Cin <= 3, K*K <= 9,
// Cout a multiple of 32. DCN_FLAG_NO_TF32 keeps such layers on CUDA cores.
bool use_fwd_f32_tc(const dcn_params_t* p, const dcn::Shape& s) {
    return p->dtype == DCN_F32 && !(p->flags & (DCN_FLAG_GENERIC | DCN_FLAG_NO_TF32)) && dcn::fwd_f32_tc_supported(s);
}

// The small-channel float32 forward: Cin <= 8, Cout a multiple of 32.
bool use_fwd_small(const dcn_params_t* p, const dcn::Shape& s) {
    return p->dtype == DCN_F32 && !(p->flags & DCN_FLAG_GENERIC) && dcn::fwd_f32_small_supported(s);
}

// The tensor-core weight gradient: bfloat16, channel counts multiples of 8, Cout <= 256.
bool use_bwd_weight_tc(const dcn_params_t* p, const dcn::Shape& s) {
    return p->dtype == DCN_BF16 && !(p->flags & DCN_FLAG_GENERIC) && dcn::bwd_weight_tc_supported(s);
}

// The tensor-core data-side backward: bfloat16, channel counts multiples of 8.
bool use_bwd_data_tc(const dcn_params_t* p, const dcn::Shape& s) {
    return p->dtype == DCN_BF16 && !(p->flags & DCN_FLAG_GENERIC) && dcn::bwd_data_tc_supported(s);
}

#define TRY(expr)                    \
    do {                             \
        int _rc = (expr);            \
        if (_rc != DCN_OK) return _rc; \
    } while (0)

}  // namespace

extern "C" {

int dcn_abi_version(void) { return DCN_ABI_VERSION; }

int dcn_output_size(const dcn_params_t* params, int* Ho, int* Wo) {
    dcn::Shape s;
    TRY(make_shape(params, s));
    if (Ho) *Ho = s.Ho;
    if (Wo) *Wo = s.Wo;
    return ok();
}

size_t dcn_workspace_size(const dcn_params_t* params, int op) {
    dcn::Shape s;
    std::string keep = g_err;
    if (make_shape(params, s) != DCN_OK) {
        g_err = keep;
        return 0;
    }
    if (op == DCN_OP_FORWARD && use_fwd_tc(params, s)) return dcn::fwd_tc_workspace(s);
    if (op == DCN_OP_BACKWARD_WEIGHT && use_bwd_weight_tc(params, s)) return dcn::bwd_weight_tc_workspace(s);
    if (op == DCN_OP_BACKWARD_DATA && use_bwd_data_tc(params, s)) return dcn::bwd_data_tc_workspace(s);
    return 0;
}

const char* dcn_forward_path(const dcn_params_t* params) {
    dcn::Shape s;
    std::string keep = g_err;
    if (make_shape(params, s) != DCN_OK) {
        g_err = keep;
        return "invalid";
    }
    if (use_fwd_tc(params, s)) return dcn::fwd_tc_variant(s);
    if (use_fwd_f32_tc(params, s)) return "tcgen05_tf32_split";
    if (use_fwd_small(params, s)) return "f32_small_channels";
    return "generic";
}

int dcn_forward(const dcn_params_t* params, const void* x, const void* offset, const void* mask, const void* weight,
                const void* bias, void* y, void* workspace, size_t workspace_bytes, void* stream) {
    DCN_TRACE("dcn_forward");
    dcn::Shape s;
    TRY(make_shape(params, s));
    size_t es = elem_size(params->dtype);
    TRY(check_ptr(x, "x", es, true));
    TRY(check_ptr(offset, "offset", es, true));
    TRY(check_ptr(mask, "mask", es, false));
    TRY(check_ptr(weight, "weight", es, true));
    TRY(check_ptr(bias, "bias", es, false));
    TRY(check_ptr(y, "y", es, true));
    cudaStream_t st = (cudaStream_t)stream;
    if (use_fwd_tc(params, s) && aligned16(x) && aligned16(weight) && aligned16(y)) {
        size_t need = dcn::fwd_tc_workspace(s);
        if (!workspace || workspace_bytes < need)
            return fail(DCN_ERR_WORKSPACE, "forward needs %zu bytes of workspace, got %zu", need,
                        workspace ? workspace_bytes : (size_t)0);
        unsigned* status = nullptr;
        cudaError_t e = dcn::status_word_ptr(&status);
        if (e != cudaSuccess) return cuda_fail(e, "status word");
        int n = 0;
        e = dcn::fwd_tc(s, x, offset, mask, weight, bias, y, workspace, workspace_bytes, status, st, &n);
        g_launches += n;
        if (e != cudaSuccess) return cuda_fail(e, "tensor-core forward launch");
        return ok();
    }
    if (use_fwd_f32_tc(params, s) && aligned16(y)) {
        unsigned* status = nullptr;
        cudaError_t e = dcn::status_word_ptr(&status);
        if (e != cudaSuccess) return cuda_fail(e, "status word");
        e = dcn::fwd_f32_tc(s, x, offset, mask, weight, bias, y, status, st);
        g_launches += 1;
        if (e != cudaSuccess) return cuda_fail(e, "float32 tensor-core forward launch");
        return ok();
    }
    if (use_fwd_small(params, s) && aligned16(y)) {
        cudaError_t e = dcn::fwd_f32_small(s, x, offset, mask, weight, bias, y, st);
        g_launches += 1;
        if (e != cudaSuccess) return cuda_fail(e, "small-channel forward launch");
        return ok();
    }
    cudaError_t e = dcn::generic_forward(s, params->dtype, x, offset, mask, weight, bias, y, st);
    g_launches += 1;
    if (e != cudaSuccess) return cuda_fail(e, "forward launch");
    return ok();
}

int dcn_forward_noalloc(const dcn_params_t* params, const void* x, const void* offset, const void* mask,
                        const void* weight, const void* bias, void* y, void* stream) {
    DCN_TRACE("dcn_forward_noalloc");
    dcn::Shape s;
    TRY(make_shape(params, s));
    size_t es = elem_size(params->dtype);
    TRY(check_ptr(x, "x", es, true));
    TRY(check_ptr(offset, "offset", es, true));
    TRY(check_ptr(mask, "mask", es, false));
    TRY(check_ptr(weight, "weight", es, true));
    TRY(check_ptr(bias, "bias", es, false));
    TRY(check_ptr(y, "y", es, true));
    if (use_fwd_tc(params, s) && aligned16(x) && aligned16(weight) && aligned16(y)) {
        const size_t need = dcn::fwd_tc_workspace(s), have = dcn::fwd_tc_static_scratch_bytes();
        if (need > have)
            return fail(DCN_ERR_WORKSPACE,
                        "forward without allocation needs %zu bytes of scratch; the static array holds %zu", need,
                        have);
        unsigned* status = nullptr;
        cudaError_t e = dcn::status_word_ptr(&status);
        if (e != cudaSuccess) return cuda_fail(e, "status word");
        int n = 0;
        e = dcn::fwd_tc_noalloc(s, x, offset, mask, weight, bias, y, status, (cudaStream_t)stream, &n);
        g_launches += n;
        if (e != cudaSuccess) return cuda_fail(e, "tensor-core forward (static scratch) launch");
        return ok();
    }
    // every other forward kernel needs no scratch
    return dcn_forward(params, x, offset, mask, weight, bias, y, nullptr, 0, stream);
}

int dcn_backward_data(const dcn_params_t* params, const void* x, const void* offset, const void* mask,
                      const void* weight, const void* grad_y, float* grad_x, float* grad_offset, float* grad_mask,
                      void* workspace, size_t workspace_bytes, void* stream) {
    DCN_TRACE("dcn_backward_data");
    dcn::Shape s;
    TRY(make_shape(params, s));
    size_t es = elem_size(params->dtype);
    TRY(check_ptr(x, "x", es, true));
    TRY(check_ptr(offset, "offset", es, true));
    TRY(check_ptr(mask, "mask", es, false));
    TRY(check_ptr(weight, "weight", es, true));
    TRY(check_ptr(grad_y, "grad_y", es, true));
    TRY(check_ptr(grad_x, "grad_x", 4, false));
    TRY(check_ptr(grad_offset, "grad_offset", 4, false));
    TRY(check_ptr(grad_mask, "grad_mask", 4, false));
    if (grad_mask && !mask) return fail(DCN_ERR_INVALID_ARG, "grad_mask requested but mask is NULL");
    if (!grad_x && !grad_offset && !grad_mask) return ok();
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e;
    if (use_bwd_data_tc(params, s) && aligned16(x) && aligned16(weight) && aligned16(grad_y) && aligned16(grad_x)) {
        const size_t need = dcn::bwd_data_tc_workspace(s);
        if (!workspace || workspace_bytes < need)
            return fail(DCN_ERR_WORKSPACE, "backward-data needs %zu bytes of workspace, got %zu", need,
                        workspace ? workspace_bytes : (size_t)0);
        unsigned* status = nullptr;
        e = dcn::status_word_ptr(&status);
        if (e != cudaSuccess) return cuda_fail(e, "status word");
        int n = 0;
        e = dcn::bwd_data_tc(s, x, offset, mask, weight, grad_y, grad_x, grad_offset, grad_mask, workspace,
                             workspace_bytes, status, st, &n);
        g_launches += n;
        if (e != cudaSuccess) return cuda_fail(e, "tensor-core backward-data launch");
        return ok();
    }
    if (grad_x) {
        e = cudaMemsetAsync(grad_x, 0, sizeof(float) * (size_t)s.B * s.H * s.W * s.Cin, st);
        g_launches += 1;
        if (e != cudaSuccess) return cuda_fail(e, "zeroing grad_x");
    }
    e = dcn::generic_backward_data(s, params->dtype, x, offset, mask, weight, grad_y, grad_x, grad_offset, grad_mask,
                                   st);
    g_launches += 1;
    if (e != cudaSuccess) return cuda_fail(e, "backward-data launch");
    return ok();
}

int dcn_backward_input(const dcn_params_t* params, const void* x, const void* offset, const void* mask,
                       const void* weight, const void* grad_y, float* grad_x, void* workspace, size_t workspace_bytes,
                       void* stream) {
    DCN_TRACE("dcn_backward_input");
    if (!grad_x) return fail(DCN_ERR_INVALID_ARG, "grad_x is NULL");
    return dcn_backward_data(params, x, offset, mask, weight, grad_y, grad_x, nullptr, nullptr, workspace,
                             workspace_bytes, stream);
}

int dcn_backward_offset_mask(const dcn_params_t* params, const void* x, const void* offset, const void* mask,
                             const void* weight, const void* grad_y, float* grad_offset, float* grad_mask,
                             void* workspace, size_t workspace_bytes, void* stream) {
    DCN_TRACE("dcn_backward_offset_mask");
    if (!grad_offset) return fail(DCN_ERR_INVALID_ARG, "grad_offset is NULL");
    return dcn_backward_data(params, x, offset, mask, weight, grad_y, nullptr, grad_offset, grad_mask, workspace,
                             workspace_bytes, stream);
}

int dcn_backward_weight(const dcn_params_t* params, const void* x, const void* offset, const void* mask,
                        const void* grad_y, float* grad_weight, float* grad_bias, void* workspace,
                        size_t workspace_bytes, void* stream) {
    DCN_TRACE("dcn_backward_weight");
    dcn::Shape s;
    TRY(make_shape(params, s));
    size_t es = elem_size(params->dtype);
    TRY(check_ptr(x, "x", es, true));
    TRY(check_ptr(offset, "offset", es, true));
    TRY(check_ptr(mask, "mask", es, false));
    TRY(check_ptr(grad_y, "grad_y", es, true));
    TRY(check_ptr(grad_weight, "grad_weight", 4, true));
    TRY(check_ptr(grad_bias, "grad_bias", 4, false));
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e;
    if (grad_bias) {  // zeroed first, so that its kernel can follow the weight kernel's launch directly
        e = cudaMemsetAsync(grad_bias, 0, sizeof(float) * (size_t)s.Cout, st);
        g_launches += 1;
        if (e != cudaSuccess) return cuda_fail(e, "zeroing grad_bias");
    }
    bool tc = false;
    if (use_bwd_weight_tc(params, s) && aligned16(x) && aligned16(grad_y) && aligned16(grad_weight)) {
        tc = true;
        const size_t need = dcn::bwd_weight_tc_workspace(s);
        if (!workspace || workspace_bytes < need)
            return fail(DCN_ERR_WORKSPACE, "backward-weight needs %zu bytes of workspace, got %zu", need,
                        workspace ? workspace_bytes : (size_t)0);
        unsigned* status = nullptr;
        e = dcn::status_word_ptr(&status);
        if (e != cudaSuccess) return cuda_fail(e, "status word");
        int n = 0;
        e = dcn::bwd_weight_tc(s, x, offset, mask, grad_y, grad_weight, workspace, workspace_bytes, status, st, &n);
        g_launches += n;
        if (e != cudaSuccess) return cuda_fail(e, "tensor-core backward-weight launch");
    } else {
        e = cudaMemsetAsync(grad_weight, 0, sizeof(float) * (size_t)s.Cout * s.KC, st);
        g_launches += 1;
        if (e != cudaSuccess) return cuda_fail(e, "zeroing grad_weight");
        e = dcn::generic_backward_weight(s, params->dtype, x, offset, mask, grad_y, grad_weight, st);
        g_launches += 1;
        if (e != cudaSuccess) return cuda_fail(e, "backward-weight launch");
    }
    if (grad_bias) {
        // after the tensor-core weight kernel: a programmatic dependent that runs alongside it
        e = dcn::bias_grad(s, params->dtype, grad_y, grad_bias, st, tc);
        g_launches += 1;
        if (e != cudaSuccess) return cuda_fail(e, "bias-gradient launch");
    }
    return ok();
}

// ------------------------------------------------- offset/mask predictor --

// The predictor is the plain convolution with the layer's kernel size, stride,
// padding and dilation and 3*G*K*K outputs. bfloat16 layers of stride 1 run it
// as one tensor-core kernel (no workspace); the others run it as this library's
// layer with zero offsets, no mask, one group and the outputs padded to a
// multiple of 32, then split the result. Workspace pieces of that path, each
// 256-byte aligned: the zero offsets, the padded weights and bias, the [P, NP]
// result, and the inner forward's own workspace.
struct PredPlan {
    dcn_params_t q;   // the inner plain convolution
    int nc, np, no;   // 3GK^2 outputs, rounded up to 32, of which 2GK^2 offsets
    size_t zoff, wpad, bpad, ypred, fws, fws_bytes, total;
};

static int pred_plan(const dcn_params_t* p, PredPlan& pl, dcn::Shape& s) {
    if (!p) return fail(DCN_ERR_INVALID_ARG, "params is NULL");
    dcn_params_t lay = *p;
    lay.Cout = 1;  // the layer's Cout plays no part in the predictor
    TRY(make_shape(&lay, s));
    pl.nc = 3 * p->G * s.K2;
    pl.no = 2 * p->G * s.K2;
    pl.np = (pl.nc + 31) / 32 * 32;
    pl.q = lay;
    pl.q.Cout = pl.np;
    pl.q.G = 1;
    dcn::Shape sq;
    TRY(make_shape(&pl.q, sq));
    const size_t es = elem_size(p->dtype);
    auto up = [](size_t v) { return (v + 255) & ~(size_t)255; };
    size_t o = 0;
    pl.zoff = o;
    o = up(o + es * (size_t)s.P * 2 * s.K2);
    pl.wpad = o;
    o = up(o + es * (size_t)pl.np * s.KC);
    pl.bpad = o;
    o = up(o + es * (size_t)pl.np);
    pl.ypred = o;
    o = up(o + es * (size_t)s.P * pl.np);
    pl.fws = o;
    pl.fws_bytes = dcn_workspace_size(&pl.q, DCN_OP_FORWARD);
    pl.total = up(o + pl.fws_bytes);
    return DCN_OK;
}

static bool use_pred_tc(const dcn_params_t* p, const dcn::Shape& s) {
    return p->dtype == DCN_BF16 && !(p->flags & DCN_FLAG_GENERIC) && dcn::pred_tc_supported(s);
}

size_t dcn_predict_workspace_size(const dcn_params_t* params) {
    PredPlan pl;
    dcn::Shape s;
    std::string keep = g_err;
    if (pred_plan(params, pl, s) != DCN_OK) {
        g_err = keep;
        return 0;
    }
    return use_pred_tc(params, s) ? 0 : pl.total;
}

int dcn_predict_offset_mask(const dcn_params_t* params, const void* x, const void* w_pred, const void* b_pred,
                            void* offset, void* mask, void* workspace, size_t workspace_bytes, void* stream) {
    DCN_TRACE("dcn_predict_offset_mask");
    PredPlan pl;
    dcn::Shape s;
    TRY(pred_plan(params, pl, s));
    const size_t es = elem_size(params->dtype);
    TRY(check_ptr(x, "x", es, true));
    TRY(check_ptr(w_pred, "w_pred", es, true));
    TRY(check_ptr(b_pred, "b_pred", es, false));
    TRY(check_ptr(offset, "offset", es, true));
    TRY(check_ptr(mask, "mask", es, true));
    cudaStream_t st = (cudaStream_t)stream;
    if (use_pred_tc(params, s)) {
        // the tensor maps of x and w_pred need 16-byte aligned bases
        if (!aligned16(x) || !aligned16(w_pred))
            return fail(DCN_ERR_UNSUPPORTED, "x and w_pred must be 16-byte aligned for this layer");
        unsigned* status = nullptr;
        cudaError_t e = dcn::status_word_ptr(&status);
        if (e != cudaSuccess) return cuda_fail(e, "status word");
        e = dcn::pred_tc(s, x, w_pred, b_pred, offset, mask, status, st);
        g_launches += 1;
        if (e != cudaSuccess) return cuda_fail(e, "tensor-core predictor launch");
        return ok();
    }
    if (!workspace || workspace_bytes < pl.total)
        return fail(DCN_ERR_WORKSPACE, "the predictor needs %zu bytes of workspace, got %zu", pl.total,
                    workspace ? workspace_bytes : (size_t)0);
    TRY(check_ptr(workspace, "workspace", 256, true));
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const int bf = params->dtype == DCN_BF16;
    cudaError_t e = cudaMemsetAsync(ws + pl.zoff, 0, es * (size_t)s.P * 2 * s.K2, st);
    g_launches += 1;
    if (e != cudaSuccess) return cuda_fail(e, "zeroing the predictor's offsets");
    e = dcn::predict_pad(bf, w_pred, b_pred, ws + pl.wpad, ws + pl.bpad, pl.nc, pl.np, s.KC, st);
    g_launches += 1;
    if (e != cudaSuccess) return cuda_fail(e, "padding the predictor weights");
    const int rc = dcn_forward(&pl.q, x, ws + pl.zoff, nullptr, ws + pl.wpad, ws + pl.bpad, ws + pl.ypred,
                               ws + pl.fws, pl.fws_bytes, stream);
    if (rc != DCN_OK) return rc;
    e = dcn::predict_split(bf, ws + pl.ypred, offset, mask, s.P, s.Ho * s.Wo, pl.np, pl.no, pl.nc, st);
    g_launches += 1;
    if (e != cudaSuccess) return cuda_fail(e, "splitting the predictor output");
    return ok();
}

// ------------------------------------------------ deformable RoI pooling --

static int roi_args(const dcn_roi_params_t* p, dcn::RoiArgs& a, const float* rois) {
    if (!p) return fail(DCN_ERR_INVALID_ARG, "params is NULL");
    if (p->B < 1 || p->H < 1 || p->W < 1 || p->C < 1 || p->R < 0 || p->k < 1 || p->k > 64)
        return fail(DCN_ERR_INVALID_ARG,
                    "need B, H, W, C >= 1, R >= 0 and 1 <= k <= 64 (B=%d H=%d W=%d C=%d R=%d k=%d)", p->B, p->H, p->W,
                    p->C, p->R, p->k);
    if (p->dtype != DCN_F32 && p->dtype != DCN_BF16) return fail(DCN_ERR_UNSUPPORTED, "unknown dtype %d", p->dtype);
    if (!(p->gamma > -3.0e38f && p->gamma < 3.0e38f)) return fail(DCN_ERR_INVALID_ARG, "gamma must be finite");
    if ((long long)p->B * p->H * p->W * p->C > kMaxElems || (long long)p->R * p->k * p->k * p->C > kMaxElems)
        return fail(DCN_ERR_UNSUPPORTED, "a tensor exceeds 2^31-1 elements");
    a.rois = rois;
    a.B = p->B;
    a.H = p->H;
    a.W = p->W;
    a.C = p->C;
    a.R = p->R;
    a.k = p->k;
    a.gamma = p->gamma;
    return DCN_OK;
}

int dcn_droi_pool_forward(const dcn_roi_params_t* params, const void* x, const float* rois, const void* offset,
                          const void* mask, void* y, void* stream) {
    DCN_TRACE("dcn_droi_pool_forward");
    dcn::RoiArgs a;
    TRY(roi_args(params, a, rois));
    const size_t es = elem_size(params->dtype);
    const bool any = params->R > 0;
    TRY(check_ptr(x, "x", es, true));
    TRY(check_ptr(rois, "rois", 4, any));
    TRY(check_ptr(offset, "offset", es, false));
    TRY(check_ptr(mask, "mask", es, false));
    TRY(check_ptr(y, "y", es, any));
    if (!any) return ok();
    cudaError_t e = dcn::droi_forward(a, params->dtype == DCN_BF16, x, offset, mask, y, (cudaStream_t)stream);
    g_launches += 1;
    if (e != cudaSuccess) return cuda_fail(e, "RoI pooling forward launch");
    return ok();
}

int dcn_droi_pool_backward(const dcn_roi_params_t* params, const void* x, const float* rois, const void* offset,
                           const void* mask, const void* grad_y, float* grad_x, float* grad_offset, float* grad_mask,
                           void* stream) {
    DCN_TRACE("dcn_droi_pool_backward");
    dcn::RoiArgs a;
    TRY(roi_args(params, a, rois));
    const size_t es = elem_size(params->dtype);
    const bool any = params->R > 0;
    TRY(check_ptr(x, "x", es, true));
    TRY(check_ptr(rois, "rois", 4, any));
    TRY(check_ptr(offset, "offset", es, false));
    TRY(check_ptr(mask, "mask", es, false));
    TRY(check_ptr(grad_y, "grad_y", es, any));
    TRY(check_ptr(grad_x, "grad_x", 4, true));
    TRY(check_ptr(grad_offset, "grad_offset", 4, false));
    TRY(check_ptr(grad_mask, "grad_mask", 4, false));
    if (grad_offset && !offset) return fail(DCN_ERR_INVALID_ARG, "grad_offset needs offset");
    if (grad_mask && !mask) return fail(DCN_ERR_INVALID_ARG, "grad_mask needs mask");
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaMemsetAsync(grad_x, 0, sizeof(float) * (size_t)a.B * a.H * a.W * a.C, st);
    g_launches += 1;
    if (e != cudaSuccess) return cuda_fail(e, "zeroing grad_x");
    if (!any) return ok();
    e = dcn::droi_backward(a, params->dtype == DCN_BF16, x, offset, mask, grad_y, grad_x, grad_offset, grad_mask, st);
    g_launches += 1;
    if (e != cudaSuccess) return cuda_fail(e, "RoI pooling backward launch");
    return ok();
}

const char* dcn_last_error_string(void) { return g_err.c_str(); }

int dcn_check_status(void* stream) {
    DCN_TRACE("dcn_check_status");
    unsigned int st = 0;
    cudaError_t e = dcn::read_and_clear_status(&st, (cudaStream_t)stream);
    g_launches += 1;
    if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
    if (st & 2u)  // kStatusRange
        return fail(DCN_ERR_RANGE, "a device access fell outside its buffer and was skipped (status 0x%x)", st);
    if (st) return fail(DCN_ERR_TIMEOUT, "a kernel gave up a bounded wait (status 0x%x)", st);
    return ok();
}

int dcn_selftest_wait_timeout(unsigned long long limit_cycles, void* stream) {
    DCN_TRACE("dcn_selftest_wait_timeout");
    if (limit_cycles < 1000ull || limit_cycles > 4000000000ull)
        return fail(DCN_ERR_INVALID_ARG, "limit_cycles must be in [1e3, 4e9], got %llu", limit_cycles);
    cudaError_t e = dcn::selftest_wait_timeout((long long)limit_cycles, (cudaStream_t)stream);
    g_launches += 1;
    if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
    return ok();
}

unsigned long long dcn_launch_count(void) { return g_launches.load(); }

}  // extern "C"
