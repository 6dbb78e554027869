"""Float64 CPU oracle for the modulated deformable convolution (DCNv2).

TEST INFRASTRUCTURE ONLY. The oracle is what the CUDA library is checked
against; only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` may import it. The product never calls it, and the two share no
code: this package wraps a plain C loop nest (``dcn_oracle.c``) through ctypes
and takes numpy float64 arrays in the layouts documented there.

What it computes follows the pages' definitions (cited function by function in
``dcn_oracle.c``):

* the deformable convolution y(p0) = sum_k w(p_k) * x(p0 + p_k + dp_k) with
  bilinear sampling ("Deformable ConvNets" notes, "可变形卷积" equations and the
  "双线性插值" S1..S4 weights),
* the DCNv2 modulation scalar per tap ("DCNv2", section 3.2),
* deformable groups (notes, "Deformable Group"),
* torchvision ``deform_conv2d`` layout and zero contribution from neighbours
  outside the map (tutorial, section 2).

Parity is pinned by ``tests/test_oracle_pins.py`` against facts that do not
come from the oracle itself (a direct convolution, shifted convolutions, closed
forms of bilinear sampling, adjoint identities, finite differences).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dcn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_dcn.so")
_lock = threading.Lock()
_lib = None


class Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "H", "W", "Cin", "Cout", "K", "stride", "pad", "dil", "G")]


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle with gcc (C99, -O2, OpenMP, no FP contraction)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-shared", "-fPIC",
               "-o", tmp, src, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, out)
    return out


def load(path: str | None = None):
    """Load (building if needed) the oracle library; returns the ctypes handle."""
    global _lib
    with _lock:
        if path is not None:
            return _bind(ctypes.CDLL(path))
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
        return _lib


def _bind(lib):
    dp = ctypes.POINTER(ctypes.c_double)
    lp = ctypes.POINTER(ctypes.c_long)
    sp = ctypes.POINTER(Shape)
    L = ctypes.c_long
    lib.dcn_oracle_out_h.argtypes = [sp]
    lib.dcn_oracle_out_w.argtypes = [sp]
    lib.dcn_oracle_set_threads.argtypes = [ctypes.c_int]
    lib.dcn_oracle_max_threads.restype = ctypes.c_int
    lib.dcn_oracle_forward.argtypes = [sp, dp, dp, dp, dp, dp, dp]
    lib.dcn_oracle_forward_pixels.argtypes = [sp, dp, dp, dp, dp, dp, L, lp, dp]
    lib.dcn_oracle_bilinear.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, dp, ctypes.c_double,
                                        ctypes.c_double, dp]
    lib.dcn_oracle_backward.argtypes = [sp, dp, dp, dp, dp, dp, dp, dp, dp, dp, dp]
    lib.dcn_oracle_grad_offset_mask_pixels.argtypes = [sp, dp, dp, dp, dp, dp, L, lp, dp, dp]
    lib.dcn_oracle_grad_weight_entries.argtypes = [sp, dp, dp, dp, dp, L, lp, dp]
    lib.dcn_oracle_grad_x_entries.argtypes = [sp, dp, dp, dp, dp, L, lp, dp]
    lib.dcn_oracle_predict_offset_mask.argtypes = [sp, dp, dp, dp, dp, dp]
    I, D = ctypes.c_int, ctypes.c_double
    lib.dcn_oracle_droi_pool_forward.argtypes = [sp, I, I, D, dp, dp, dp, dp, dp]
    lib.dcn_oracle_droi_pool_backward.argtypes = [sp, I, I, D, dp, dp, dp, dp, dp, dp, dp, dp]
    return lib


def _d(a):
    """float64 C-contiguous view/copy of an array-like, or NULL for None."""
    if a is None:
        return None, None
    arr = np.ascontiguousarray(np.asarray(a, dtype=np.float64))
    return arr, arr.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _shape(B, H, W, Cin, Cout, K, stride=1, pad=0, dil=1, G=1):
    return Shape(B, H, W, Cin, Cout, K, stride, pad, dil, G)


def out_hw(H, W, K, stride=1, pad=0, dil=1, lib=None):
    lib = lib or load()
    s = _shape(1, H, W, 1, 1, K, stride, pad, dil, 1)
    return lib.dcn_oracle_out_h(ctypes.byref(s)), lib.dcn_oracle_out_w(ctypes.byref(s))


def set_threads(n: int, lib=None):
    (lib or load()).dcn_oracle_set_threads(int(n))


def max_threads(lib=None) -> int:
    return int((lib or load()).dcn_oracle_max_threads())


def _dims(x, weight, offset, G):
    B, H, W, Cin = x.shape
    Cout, K, K2, Cw = weight.shape
    assert K == K2 and Cw == Cin, "weight must be [Cout, K, K, Cin]"
    return B, H, W, Cin, Cout, K


def forward(x, offset, mask, weight, bias=None, stride=1, pad=0, dil=1, G=1, pixels=None, lib=None):
    """y [B, Ho, Wo, Cout] (or [len(pixels), Cout] at listed flat output pixels)."""
    lib = lib or load()
    B, H, W, Cin, Cout, K = _dims(x, weight, offset, G)
    s = _shape(B, H, W, Cin, Cout, K, stride, pad, dil, G)
    Ho, Wo = lib.dcn_oracle_out_h(ctypes.byref(s)), lib.dcn_oracle_out_w(ctypes.byref(s))
    xs, xp = _d(x)
    os_, op = _d(offset)
    ms, mp = _d(mask)
    ws, wp = _d(weight)
    bs, bp = _d(bias)
    assert os_.shape == (B, 2 * G * K * K, Ho, Wo), os_.shape
    if ms is not None:
        assert ms.shape == (B, G * K * K, Ho, Wo), ms.shape
    if pixels is None:
        y = np.zeros((B, Ho, Wo, Cout))
        rc = lib.dcn_oracle_forward(ctypes.byref(s), xp, op, mp, wp, bp, y.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    else:
        pix = np.ascontiguousarray(np.asarray(pixels, dtype=np.int64))
        y = np.zeros((len(pix), Cout))
        rc = lib.dcn_oracle_forward_pixels(ctypes.byref(s), xp, op, mp, wp, bp, len(pix),
                                           pix.ctypes.data_as(ctypes.POINTER(ctypes.c_long)),
                                           y.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    if rc != 0:
        raise ValueError("oracle forward rejected the shape (rc=%d)" % rc)
    return y


def bilinear(img, py, px, lib=None):
    """Bilinear sample of an [H, W, C] image at fractional (py, px): C values."""
    lib = lib or load()
    im, ip = _d(img)
    H, W, C = im.shape
    out = np.zeros(C)
    lib.dcn_oracle_bilinear(H, W, C, ip, float(py), float(px), out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    return out


def backward(x, offset, mask, weight, grad_y, stride=1, pad=0, dil=1, G=1, lib=None):
    """Full backward: dict with grad_x, grad_offset, grad_mask (None without mask), grad_weight, grad_bias."""
    lib = lib or load()
    B, H, W, Cin, Cout, K = _dims(x, weight, offset, G)
    s = _shape(B, H, W, Cin, Cout, K, stride, pad, dil, G)
    Ho, Wo = lib.dcn_oracle_out_h(ctypes.byref(s)), lib.dcn_oracle_out_w(ctypes.byref(s))
    xs, xp = _d(x)
    os_, op = _d(offset)
    ms, mp = _d(mask)
    ws, wp = _d(weight)
    gs, gp = _d(grad_y)
    assert gs.shape == (B, Ho, Wo, Cout)
    out = {
        "grad_x": np.zeros((B, H, W, Cin)),
        "grad_offset": np.zeros((B, 2 * G * K * K, Ho, Wo)),
        "grad_mask": np.zeros((B, G * K * K, Ho, Wo)) if ms is not None else None,
        "grad_weight": np.zeros((Cout, K, K, Cin)),
        "grad_bias": np.zeros(Cout),
    }
    P = lambda a: None if a is None else a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))
    rc = lib.dcn_oracle_backward(ctypes.byref(s), xp, op, mp, wp, gp, P(out["grad_x"]), P(out["grad_offset"]),
                                 P(out["grad_mask"]), P(out["grad_weight"]), P(out["grad_bias"]))
    if rc != 0:
        raise ValueError("oracle backward failed (rc=%d)" % rc)
    return out


def grad_offset_mask_at(x, offset, mask, weight, grad_y, pixels, stride=1, pad=0, dil=1, G=1, lib=None):
    """(grad_offset [n, 2GK^2], grad_mask [n, GK^2] or None) at listed flat output pixels."""
    lib = lib or load()
    B, H, W, Cin, Cout, K = _dims(x, weight, offset, G)
    s = _shape(B, H, W, Cin, Cout, K, stride, pad, dil, G)
    xs, xp = _d(x)
    os_, op = _d(offset)
    ms, mp = _d(mask)
    ws, wp = _d(weight)
    gs, gp = _d(grad_y)
    pix = np.ascontiguousarray(np.asarray(pixels, dtype=np.int64))
    goff = np.zeros((len(pix), 2 * G * K * K))
    gm = np.zeros((len(pix), G * K * K)) if ms is not None else None
    rc = lib.dcn_oracle_grad_offset_mask_pixels(
        ctypes.byref(s), xp, op, mp, wp, gp, len(pix), pix.ctypes.data_as(ctypes.POINTER(ctypes.c_long)),
        goff.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
        None if gm is None else gm.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    if rc != 0:
        raise ValueError("oracle rc=%d" % rc)
    return goff, gm


def grad_weight_at(x, offset, mask, grad_y, weight_shape, entries, stride=1, pad=0, dil=1, G=1, lib=None):
    """grad_weight at listed flat indices into [Cout, K, K, Cin]."""
    lib = lib or load()
    B, H, W, Cin = np.shape(x)
    Cout, K = weight_shape[0], weight_shape[1]
    s = _shape(B, H, W, Cin, Cout, K, stride, pad, dil, G)
    xs, xp = _d(x)
    os_, op = _d(offset)
    ms, mp = _d(mask)
    gs, gp = _d(grad_y)
    idx = np.ascontiguousarray(np.asarray(entries, dtype=np.int64))
    out = np.zeros(len(idx))
    rc = lib.dcn_oracle_grad_weight_entries(ctypes.byref(s), xp, op, mp, gp, len(idx),
                                            idx.ctypes.data_as(ctypes.POINTER(ctypes.c_long)),
                                            out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    if rc != 0:
        raise ValueError("oracle rc=%d" % rc)
    return out


def grad_x_at(x_shape, offset, mask, weight, grad_y, entries, stride=1, pad=0, dil=1, G=1, lib=None):
    """grad_x at listed flat indices into [B, H, W, Cin]."""
    lib = lib or load()
    B, H, W, Cin = x_shape
    Cout, K = np.shape(weight)[0], np.shape(weight)[1]
    s = _shape(B, H, W, Cin, Cout, K, stride, pad, dil, G)
    os_, op = _d(offset)
    ms, mp = _d(mask)
    ws, wp = _d(weight)
    gs, gp = _d(grad_y)
    idx = np.ascontiguousarray(np.asarray(entries, dtype=np.int64))
    out = np.zeros(len(idx))
    rc = lib.dcn_oracle_grad_x_entries(ctypes.byref(s), op, mp, wp, gp, len(idx),
                                       idx.ctypes.data_as(ctypes.POINTER(ctypes.c_long)),
                                       out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    if rc != 0:
        raise ValueError("oracle rc=%d" % rc)
    return out


def predict_offset_mask(x, w_pred, b_pred, K, stride=1, pad=0, dil=1, G=1, lib=None):
    """(offset [B, 2GK^2, Ho, Wo], mask [B, GK^2, Ho, Wo]) of a DCNv2 layer from its
    predictor convolution w_pred [3GK^2, K, K, Cin] (+ b_pred [3GK^2] or None)."""
    lib = lib or load()
    B, H, W, Cin = x.shape
    assert tuple(w_pred.shape) == (3 * G * K * K, K, K, Cin), w_pred.shape
    s = _shape(B, H, W, Cin, 3 * G * K * K, K, stride, pad, dil, G)
    Ho, Wo = lib.dcn_oracle_out_h(ctypes.byref(s)), lib.dcn_oracle_out_w(ctypes.byref(s))
    xs, xp = _d(x)
    ws, wp = _d(w_pred)
    bs, bp = _d(b_pred)
    off = np.zeros((B, 2 * G * K * K, Ho, Wo))
    mask = np.zeros((B, G * K * K, Ho, Wo))
    rc = lib.dcn_oracle_predict_offset_mask(ctypes.byref(s), xp, wp, bp, off.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                                            mask.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    if rc != 0:
        raise ValueError("oracle predictor rejected the shape (rc=%d)" % rc)
    return off, mask


def droi_pool_forward(x, rois, offset, mask, k, gamma=1.0, lib=None):
    """(Modulated) deformable RoI pooling: y [R, k, k, C] from x [B, H, W, C],
    rois [R, 5] = (b, x1, y1, x2, y2), offset [R, 2k^2] (normalised, or None)
    and mask [R, k^2] (or None)."""
    lib = lib or load()
    B, H, W, C = x.shape
    R = int(np.asarray(rois).shape[0])
    s = _shape(B, H, W, C, 1, 1)
    xs, xp = _d(x)
    rs, rp = _d(rois)
    os_, op = _d(offset)
    ms, mp = _d(mask)
    y = np.zeros((R, k, k, C))
    rc = lib.dcn_oracle_droi_pool_forward(ctypes.byref(s), R, int(k), float(gamma), xp, rp, op, mp,
                                          y.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    if rc != 0:
        raise ValueError("oracle RoI pooling: a batch index is out of range")
    return y


def droi_pool_backward(x, rois, offset, mask, grad_y, k, gamma=1.0, lib=None):
    """(grad_x [B, H, W, C], grad_offset [R, 2k^2] or None, grad_mask [R, k^2] or None)."""
    lib = lib or load()
    B, H, W, C = x.shape
    R = int(np.asarray(rois).shape[0])
    s = _shape(B, H, W, C, 1, 1)
    xs, xp = _d(x)
    rs, rp = _d(rois)
    os_, op = _d(offset)
    ms, mp = _d(mask)
    gs, gp = _d(grad_y)
    gx = np.zeros((B, H, W, C))
    goff = np.zeros((R, 2 * k * k)) if offset is not None else None
    gm = np.zeros((R, k * k)) if mask is not None else None
    P = ctypes.POINTER(ctypes.c_double)
    rc = lib.dcn_oracle_droi_pool_backward(ctypes.byref(s), R, int(k), float(gamma), xp, rp, op, mp, gp,
                                           gx.ctypes.data_as(P), None if goff is None else goff.ctypes.data_as(P),
                                           None if gm is None else gm.ctypes.data_as(P))
    if rc != 0:
        raise ValueError("oracle RoI pooling: a batch index is out of range")
    return gx, goff, gm
