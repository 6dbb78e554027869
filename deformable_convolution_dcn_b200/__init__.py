"""Python binding of libdcn_b200, the sm_100a CUDA library for the modulated
deformable convolution (DCNv2, torchvision ``deform_conv2d`` semantics).

This module only marshals arguments: it checks torch CUDA tensors, passes
their device pointers and the current CUDA stream to the C ABI declared in
``include/dcn.h``, and raises on a non-zero status. Every step of the
computation runs in the library's CUDA kernels; there is no CPU fallback, and
importing works without the library but every call fails loudly until
``python -m deformable_convolution_dcn_b200.build`` has produced
``libdcn_b200.so``.

Layouts (see ``include/dcn.h``): x [B, H, W, Cin], offset [B, 2*G*K*K, Ho, Wo]
(channel g*2K^2 + 2k = row offset, +1 = column offset), mask [B, G*K*K, Ho, Wo],
weight [Cout, K, K, Cin], bias [Cout], y [B, Ho, Wo, Cout]; gradients float32.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

import torch

__all__ = [
    "forward", "forward_noalloc", "backward_data", "backward_input", "backward_offset_mask", "backward_weight", "output_size",
    "workspace_size", "forward_path", "check_status", "launch_count", "library_path", "DeformConv2dFunction",
    "deform_conv2d", "DcnError",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
# DCN_B200_LIB names another build of the library to load instead (e.g. the
# range-checked libdcn_b200_checked.so); it must sit in this package directory.
_LIB_NAME = os.environ.get("DCN_B200_LIB", "libdcn_b200.so")
if os.path.basename(_LIB_NAME) != _LIB_NAME or not _LIB_NAME.startswith("libdcn_b200"):
    raise ImportError("DCN_B200_LIB must name a libdcn_b200*.so file of the package directory, got %r" % _LIB_NAME)
_LIB_PATH = os.path.join(_PKG, _LIB_NAME)
_HEADER = os.path.join(os.path.dirname(_PKG), "include", "dcn.h")
_lock = threading.Lock()
_lib = None

DCN_F32, DCN_BF16 = 0, 1
DCN_FLAG_GENERIC = 0x1
DCN_FLAG_NO_TF32 = 0x2
DCN_ERR_TIMEOUT, DCN_ERR_RANGE = -4, -6
OP_FORWARD, OP_BACKWARD_DATA, OP_BACKWARD_WEIGHT = 0, 1, 2
_DTYPES = {torch.float32: DCN_F32, torch.bfloat16: DCN_BF16}


class DcnError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__("libdcn_b200 error %d: %s" % (code, message))
        self.code = code


class Params(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "H", "W", "Cin", "Cout", "K", "stride", "pad", "dil", "G",
                                            "dtype")] + [("flags", ctypes.c_uint)]


class RoiParams(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "H", "W", "C", "R", "k")] + [
        ("gamma", ctypes.c_float), ("dtype", ctypes.c_int), ("flags", ctypes.c_uint)]


def library_path() -> str:
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError("libdcn_b200.so is not built (expected at %s); run "
                               "`python -m deformable_convolution_dcn_b200.build`" % _LIB_PATH)
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.POINTER(Params)
        vp, fp, sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t
        lib.dcn_abi_version.restype = ctypes.c_int
        lib.dcn_output_size.argtypes = [P, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]
        lib.dcn_workspace_size.argtypes = [P, ctypes.c_int]
        lib.dcn_workspace_size.restype = sz
        lib.dcn_forward.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        lib.dcn_forward_noalloc.argtypes = [P, vp, vp, vp, vp, vp, vp, vp]
        lib.dcn_backward_data.argtypes = [P, vp, vp, vp, vp, vp, fp, fp, fp, vp, sz, vp]
        lib.dcn_backward_input.argtypes = [P, vp, vp, vp, vp, vp, fp, vp, sz, vp]
        lib.dcn_backward_offset_mask.argtypes = [P, vp, vp, vp, vp, vp, fp, fp, vp, sz, vp]
        lib.dcn_backward_weight.argtypes = [P, vp, vp, vp, vp, fp, fp, vp, sz, vp]
        lib.dcn_predict_workspace_size.argtypes = [P]
        lib.dcn_predict_workspace_size.restype = sz
        lib.dcn_predict_offset_mask.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp]
        RP = ctypes.POINTER(RoiParams)
        lib.dcn_droi_pool_forward.argtypes = [RP, vp, vp, vp, vp, vp, vp]
        lib.dcn_droi_pool_backward.argtypes = [RP, vp, vp, vp, vp, vp, fp, fp, fp, vp]
        lib.dcn_selftest_wait_timeout.argtypes = [ctypes.c_ulonglong, vp]
        lib.dcn_last_error_string.restype = ctypes.c_char_p
        lib.dcn_check_status.argtypes = [vp]
        lib.dcn_check_status.restype = ctypes.c_int
        lib.dcn_launch_count.restype = ctypes.c_ulonglong
        lib.dcn_forward_path.argtypes = [P]
        lib.dcn_forward_path.restype = ctypes.c_char_p
        _lib = lib
        return lib


def header_symbols(path: str = _HEADER):
    """Names of the entry points declared in include/dcn.h."""
    return re.findall(r"^DCN_API\s+[\w\s\*]+?\b(dcn_\w+)\s*\(", open(path).read(), flags=re.M)


def _check(rc: int):
    if rc != 0:
        raise DcnError(rc, _load().dcn_last_error_string().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def make_params(B, H, W, Cin, Cout, K, stride=1, pad=0, dil=1, G=1, dtype=DCN_F32, flags=0) -> Params:
    return Params(B, H, W, Cin, Cout, K, stride, pad, dil, G, dtype, flags)


def _params(x, weight, offset, stride, padding, dilation, generic, flags=0):
    if x.dim() != 4 or weight.dim() != 4:
        raise ValueError("x must be [B, H, W, Cin] and weight [Cout, K, K, Cin]")
    B, H, W, Cin = x.shape
    Cout, K, K2, Cw = weight.shape
    if K != K2 or Cw != Cin:
        raise ValueError("weight must be [Cout, K, K, Cin] with Cin = %d, got %s" % (Cin, tuple(weight.shape)))
    if offset.dim() != 4 or offset.shape[1] % (2 * K * K):
        raise ValueError("offset must be [B, 2*G*K*K, Ho, Wo]")
    G = offset.shape[1] // (2 * K * K)
    if x.dtype not in _DTYPES:
        raise TypeError("x must be float32 or bfloat16, got %s" % x.dtype)
    return make_params(B, H, W, Cin, Cout, K, stride, padding, dilation, G, _DTYPES[x.dtype],
                       (DCN_FLAG_GENERIC if generic else 0) | flags)


def _check_tensors(dtype, device, **ts):
    for name, t in ts.items():
        if t is None:
            continue
        if not t.is_cuda or t.device != device:
            raise ValueError("%s must be a CUDA tensor on %s" % (name, device))
        if t.dtype != dtype:
            raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
        if not t.is_contiguous():
            raise ValueError("%s must be contiguous" % name)


def output_size(p: Params):
    ho, wo = ctypes.c_int(), ctypes.c_int()
    _check(_load().dcn_output_size(ctypes.byref(p), ctypes.byref(ho), ctypes.byref(wo)))
    return ho.value, wo.value


def workspace_size(p: Params, op: int) -> int:
    return int(_load().dcn_workspace_size(ctypes.byref(p), op))


def forward_path(p: Params) -> str:
    return _load().dcn_forward_path(ctypes.byref(p)).decode()


def check_status(stream=None):
    """Waits for `stream` (a torch.cuda.Stream; default: the current stream of
    the current device) and takes the device status word, raising DcnError
    (code -4, DCN_ERR_TIMEOUT) if a kernel of the library gave up a bounded wait
    since the word was last taken, or (range-checked build) code -6,
    DCN_ERR_RANGE, if a checked access fell outside its buffer. Other streams
    are not waited for."""
    s = torch.cuda.current_stream() if stream is None else stream
    _check(_load().dcn_check_status(ctypes.c_void_p(s.cuda_stream)))


def launch_count() -> int:
    return int(_load().dcn_launch_count())


def _workspace(p, op, device, workspace):
    n = workspace_size(p, op)
    if n == 0:
        return None, 0
    if workspace is not None:
        return workspace, workspace.numel() * workspace.element_size()
    return torch.empty(n, dtype=torch.uint8, device=device), n


def forward(x, offset, mask, weight, bias=None, stride=1, padding=0, dilation=1, *, out=None, workspace=None,
            generic=False, flags=0):
    """y [B, Ho, Wo, Cout] = DCNv2(x, offset, mask, weight, bias) on x's device and current stream.
    flags: extra DCN_FLAG_* bits (DCN_FLAG_NO_TF32 keeps float32 layers off the split-tf32 kernel)."""
    lib = _load()
    p = _params(x, weight, offset, stride, padding, dilation, generic, flags)
    _check_tensors(x.dtype, x.device, x=x, offset=offset, mask=mask, weight=weight, bias=bias, out=out)
    Ho, Wo = output_size(p)
    if out is None:
        out = torch.empty((p.B, Ho, Wo, p.Cout), dtype=x.dtype, device=x.device)
    ws, nws = _workspace(p, OP_FORWARD, x.device, workspace)
    _check(lib.dcn_forward(ctypes.byref(p), _ptr(x), _ptr(offset), _ptr(mask), _ptr(weight), _ptr(bias), _ptr(out),
                           _ptr(ws), nws, _stream(x.device)))
    return out


def forward_noalloc(x, offset, mask, weight, bias=None, stride=1, padding=0, dilation=1, *, out=None):
    """Forward through dcn_forward_noalloc: no workspace, scratch in the library's static device array."""
    lib = _load()
    p = _params(x, weight, offset, stride, padding, dilation, False)
    _check_tensors(x.dtype, x.device, x=x, offset=offset, mask=mask, weight=weight, bias=bias, out=out)
    Ho, Wo = output_size(p)
    if out is None:
        out = torch.empty((p.B, Ho, Wo, p.Cout), dtype=x.dtype, device=x.device)
    _check(lib.dcn_forward_noalloc(ctypes.byref(p), _ptr(x), _ptr(offset), _ptr(mask), _ptr(weight), _ptr(bias),
                                   _ptr(out), _stream(x.device)))
    return out


def predict_workspace_size(p: Params) -> int:
    return int(_load().dcn_predict_workspace_size(ctypes.byref(p)))


def predict_offset_mask(x, w_pred, b_pred, K, stride=1, padding=0, dilation=1, G=1, *, workspace=None,
                        generic=False, out=None):
    """The offsets [B, 2GK^2, Ho, Wo] and masks [B, GK^2, Ho, Wo] of a DCNv2 layer with kernel size K, stride,
    padding, dilation and G offset groups, from its predictor convolution w_pred [3GK^2, K, K, Cin]
    (+ b_pred [3GK^2] or None) over x [B, H, W, Cin]. out: optional (offset, mask) to write."""
    lib = _load()
    if x.dim() != 4 or w_pred.dim() != 4:
        raise ValueError("x must be [B, H, W, Cin] and w_pred [3*G*K*K, K, K, Cin]")
    if x.dtype not in _DTYPES:
        raise TypeError("x must be float32 or bfloat16, got %s" % x.dtype)
    B, H, W, Cin = x.shape
    if tuple(w_pred.shape) != (3 * G * K * K, K, K, Cin):
        raise ValueError("w_pred must be %s, got %s" % ((3 * G * K * K, K, K, Cin), tuple(w_pred.shape)))
    if b_pred is not None and tuple(b_pred.shape) != (3 * G * K * K,):
        raise ValueError("b_pred must be [%d]" % (3 * G * K * K))
    p = make_params(B, H, W, Cin, 1, K, stride, padding, dilation, G, _DTYPES[x.dtype],
                    DCN_FLAG_GENERIC if generic else 0)
    Ho, Wo = output_size(p)
    if out is None:
        out = (torch.empty((B, 2 * G * K * K, Ho, Wo), dtype=x.dtype, device=x.device),
               torch.empty((B, G * K * K, Ho, Wo), dtype=x.dtype, device=x.device))
    offset, mask = out
    if tuple(offset.shape) != (B, 2 * G * K * K, Ho, Wo) or tuple(mask.shape) != (B, G * K * K, Ho, Wo):
        raise ValueError("out must be (offset %s, mask %s)" % ((B, 2 * G * K * K, Ho, Wo), (B, G * K * K, Ho, Wo)))
    _check_tensors(x.dtype, x.device, x=x, w_pred=w_pred, b_pred=b_pred, offset=offset, mask=mask)
    n = predict_workspace_size(p)
    if workspace is None and n > 0:
        workspace = torch.empty(n, dtype=torch.uint8, device=x.device)
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.dcn_predict_offset_mask(ctypes.byref(p), _ptr(x), _ptr(w_pred), _ptr(b_pred), _ptr(offset),
                                       _ptr(mask), _ptr(workspace), nbytes, _stream(x.device)))
    return offset, mask


def _roi_params(x, rois, k, gamma):
    if x.dim() != 4:
        raise ValueError("x must be [B, H, W, C]")
    if x.dtype not in _DTYPES:
        raise TypeError("x must be float32 or bfloat16, got %s" % x.dtype)
    if rois.dim() != 2 or rois.shape[1] != 5 or rois.dtype != torch.float32:
        raise ValueError("rois must be a float32 [R, 5] tensor of (b, x1, y1, x2, y2)")
    B, H, W, C = x.shape
    return RoiParams(B, H, W, C, rois.shape[0], int(k), float(gamma), _DTYPES[x.dtype], 0)


def _check_roi_inputs(p, x, rois, offset, mask):
    kk = p.k * p.k
    if offset is not None and tuple(offset.shape) != (p.R, 2 * kk):
        raise ValueError("offset must be [R, 2*k*k] = %s" % ((p.R, 2 * kk),))
    if mask is not None and tuple(mask.shape) != (p.R, kk):
        raise ValueError("mask must be [R, k*k] = %s" % ((p.R, kk),))
    _check_tensors(x.dtype, x.device, x=x, offset=offset, mask=mask)
    _check_tensors(torch.float32, x.device, rois=rois)


def droi_pool_forward(x, rois, offset, mask, k, gamma=1.0, *, out=None):
    """(Modulated) deformable RoI pooling: y [R, k, k, C] from x [B, H, W, C], rois float32 [R, 5]
    = (b, x1, y1, x2, y2), offset [R, 2k^2] (normalised, or None) and mask [R, k^2] (or None)."""
    lib = _load()
    p = _roi_params(x, rois, k, gamma)
    _check_roi_inputs(p, x, rois, offset, mask)
    if out is None:
        out = torch.empty((p.R, p.k, p.k, p.C), dtype=x.dtype, device=x.device)
    if tuple(out.shape) != (p.R, p.k, p.k, p.C):
        raise ValueError("out must be [R, k, k, C]")
    _check_tensors(x.dtype, x.device, out=out)
    _check(lib.dcn_droi_pool_forward(ctypes.byref(p), _ptr(x), _ptr(rois), _ptr(offset), _ptr(mask), _ptr(out),
                                     _stream(x.device)))
    return out


def droi_pool_backward(x, rois, offset, mask, grad_y, k, gamma=1.0, *, need_offset=True, need_mask=True):
    """(grad_x [B, H, W, C], grad_offset [R, 2k^2] or None, grad_mask [R, k^2] or None), float32."""
    lib = _load()
    p = _roi_params(x, rois, k, gamma)
    _check_roi_inputs(p, x, rois, offset, mask)
    _check_tensors(x.dtype, x.device, grad_y=grad_y)
    f32 = dict(dtype=torch.float32, device=x.device)
    gx = torch.empty(tuple(x.shape), **f32)
    goff = torch.empty((p.R, 2 * p.k * p.k), **f32) if (need_offset and offset is not None) else None
    gm = torch.empty((p.R, p.k * p.k), **f32) if (need_mask and mask is not None) else None
    _check(lib.dcn_droi_pool_backward(ctypes.byref(p), _ptr(x), _ptr(rois), _ptr(offset), _ptr(mask), _ptr(grad_y),
                                      _ptr(gx), _ptr(goff), _ptr(gm), _stream(x.device)))
    return gx, goff, gm


def backward_data(x, offset, mask, weight, grad_y, stride=1, padding=0, dilation=1, *, need_input=True,
                  need_offset=True, need_mask=True, workspace=None, generic=False, out=None):
    """(grad_x, grad_offset, grad_mask) in one pass; entries not requested are None."""
    lib = _load()
    p = _params(x, weight, offset, stride, padding, dilation, generic)
    _check_tensors(x.dtype, x.device, x=x, offset=offset, mask=mask, weight=weight, grad_y=grad_y)
    f32 = dict(dtype=torch.float32, device=x.device)
    gx, goff, gm = out if out is not None else (
        torch.empty(x.shape, **f32) if need_input else None,
        torch.empty(offset.shape, **f32) if need_offset else None,
        torch.empty(mask.shape, **f32) if (need_mask and mask is not None) else None)
    ws, nws = _workspace(p, OP_BACKWARD_DATA, x.device, workspace)
    _check(lib.dcn_backward_data(ctypes.byref(p), _ptr(x), _ptr(offset), _ptr(mask), _ptr(weight), _ptr(grad_y),
                                 _ptr(gx), _ptr(goff), _ptr(gm), _ptr(ws), nws, _stream(x.device)))
    return gx, goff, gm


def backward_input(x, offset, mask, weight, grad_y, stride=1, padding=0, dilation=1, *, workspace=None,
                   generic=False):
    lib = _load()
    p = _params(x, weight, offset, stride, padding, dilation, generic)
    _check_tensors(x.dtype, x.device, x=x, offset=offset, mask=mask, weight=weight, grad_y=grad_y)
    gx = torch.empty(x.shape, dtype=torch.float32, device=x.device)
    ws, nws = _workspace(p, OP_BACKWARD_DATA, x.device, workspace)
    _check(lib.dcn_backward_input(ctypes.byref(p), _ptr(x), _ptr(offset), _ptr(mask), _ptr(weight), _ptr(grad_y),
                                  _ptr(gx), _ptr(ws), nws, _stream(x.device)))
    return gx


def backward_offset_mask(x, offset, mask, weight, grad_y, stride=1, padding=0, dilation=1, *, workspace=None,
                         generic=False):
    lib = _load()
    p = _params(x, weight, offset, stride, padding, dilation, generic)
    _check_tensors(x.dtype, x.device, x=x, offset=offset, mask=mask, weight=weight, grad_y=grad_y)
    goff = torch.empty(offset.shape, dtype=torch.float32, device=x.device)
    gm = None if mask is None else torch.empty(mask.shape, dtype=torch.float32, device=x.device)
    ws, nws = _workspace(p, OP_BACKWARD_DATA, x.device, workspace)
    _check(lib.dcn_backward_offset_mask(ctypes.byref(p), _ptr(x), _ptr(offset), _ptr(mask), _ptr(weight),
                                        _ptr(grad_y), _ptr(goff), _ptr(gm), _ptr(ws), nws, _stream(x.device)))
    return goff, gm


def backward_weight(x, offset, mask, grad_y, weight_shape, stride=1, padding=0, dilation=1, *, need_bias=True,
                    workspace=None, generic=False, out=None):
    """(grad_weight [Cout, K, K, Cin], grad_bias [Cout] or None)."""
    lib = _load()
    wmeta = torch.empty(weight_shape, dtype=x.dtype, device="meta")
    p = _params(x, wmeta, offset, stride, padding, dilation, generic)
    _check_tensors(x.dtype, x.device, x=x, offset=offset, mask=mask, grad_y=grad_y)
    f32 = dict(dtype=torch.float32, device=x.device)
    gw, gb = out if out is not None else (torch.empty(weight_shape, **f32),
                                          torch.empty((weight_shape[0],), **f32) if need_bias else None)
    ws, nws = _workspace(p, OP_BACKWARD_WEIGHT, x.device, workspace)
    _check(lib.dcn_backward_weight(ctypes.byref(p), _ptr(x), _ptr(offset), _ptr(mask), _ptr(grad_y), _ptr(gw),
                                   _ptr(gb), _ptr(ws), nws, _stream(x.device)))
    return gw, gb


class DeformConv2dFunction(torch.autograd.Function):
    """Autograd wrapper over the library's forward and backward entry points.

    Gradients are float32 (the library's contract) and are cast to each
    input's dtype on return.
    """

    @staticmethod
    def forward(ctx, x, offset, mask, weight, bias, stride, padding, dilation):
        ctx.save_for_backward(x, offset, mask, weight)
        ctx.conf = (stride, padding, dilation, bias is not None)
        return forward(x, offset, mask, weight, bias, stride, padding, dilation)

    @staticmethod
    def backward(ctx, grad_y):
        x, offset, mask, weight = ctx.saved_tensors
        stride, padding, dilation, has_bias = ctx.conf
        gy = grad_y.contiguous().to(x.dtype)
        gx, goff, gm = backward_data(x, offset, mask, weight, gy, stride, padding, dilation)
        gw, gb = backward_weight(x, offset, mask, gy, tuple(weight.shape), stride, padding, dilation,
                                 need_bias=has_bias)
        cast = lambda g, ref: None if g is None else g.to(ref.dtype)
        return (cast(gx, x), cast(goff, offset), None if mask is None else cast(gm, mask), cast(gw, weight),
                None if gb is None else gb.to(weight.dtype), None, None, None)


def deform_conv2d(x, offset, weight, bias=None, stride=1, padding=0, dilation=1, mask=None):
    """Differentiable DCNv2 on NHWC x; argument order as torchvision's deform_conv2d."""
    return DeformConv2dFunction.apply(x, offset, mask, weight, bias, stride, padding, dilation)
