"""Helpers shared by the GPU parity tests: run the CUDA library through the
Python binding (which calls the C ABI) and compare with the float64 oracle.

Tolerances (fixed per path, not tuned to results):
  * float32 path: elementwise |gpu - ref| <= 1e-4 * (1 + |ref|);
  * bfloat16-in / float32-accumulate path: normwise ||gpu - ref||_2 / ||ref||_2 <= 1e-2
    per output tensor.
The oracle always reads the exact values the GPU reads (bfloat16 inputs are
widened to float64), so the comparison measures the kernels' arithmetic only.
"""
from __future__ import annotations

import numpy as np
import torch

import deformable_convolution_dcn_b200 as dcn
from deformable_convolution_dcn_b200 import inputs as gen

F32_RTOL = 1e-4
BF16_NORMWISE = 1e-2


def to_dev(d, device="cuda"):
    return {k: (None if v is None else v.to(device)) for k, v in d.items()}


def f64(d):
    return {k: gen.as_f64(v) for k, v in d.items()}


def assert_close(gpu, ref, dtype, what=""):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), "%s: non-finite values" % what
    if dtype == "f32":
        err = np.abs(gpu - ref) / (1.0 + np.abs(ref))
        worst = np.unravel_index(int(np.argmax(err)), err.shape) if err.size else None
        assert err.size == 0 or err.max() <= F32_RTOL, \
            "%s: max |err|/(1+|ref|) = %.3g at %s (gpu %r, ref %r)" % (what, err.max(), worst, gpu[worst], ref[worst])
    else:
        nref = np.linalg.norm(ref)
        nerr = np.linalg.norm(gpu - ref)
        rel = nerr / nref if nref > 0 else nerr
        assert rel <= BF16_NORMWISE, "%s: normwise error %.3g" % (what, rel)


def run_forward(s: gen.LayerShape, d, generic=False):
    y = dcn.forward(d["x"], d["offset"], d["mask"], d["weight"], d["bias"], s.stride, s.pad, s.dil, generic=generic)
    torch.cuda.synchronize()
    dcn.check_status()
    return y


def run_backward(s: gen.LayerShape, d, generic=False):
    gx, goff, gm = dcn.backward_data(d["x"], d["offset"], d["mask"], d["weight"], d["grad_y"], s.stride, s.pad,
                                     s.dil, generic=generic)
    gw, gb = dcn.backward_weight(d["x"], d["offset"], d["mask"], d["grad_y"], tuple(d["weight"].shape), s.stride,
                                 s.pad, s.dil, need_bias=True, generic=generic)
    torch.cuda.synchronize()
    dcn.check_status()
    return dict(grad_x=gx, grad_offset=goff, grad_mask=gm, grad_weight=gw, grad_bias=gb)


def sample_pixels(s: gen.LayerShape, n: int, seed: int):
    """Flat output-pixel indices: corners and edges of each image plus random ones."""
    r = np.random.default_rng(seed)
    plane = s.Ho * s.Wo
    fixed = []
    for b in (0, s.B - 1):
        for ho in (0, s.Ho - 1):
            for wo in (0, s.Wo // 2, s.Wo - 1):
                fixed.append(b * plane + ho * s.Wo + wo)
    rand = r.choice(s.P, size=max(0, n - len(fixed)), replace=False)
    return np.unique(np.concatenate([np.array(fixed, dtype=np.int64), rand.astype(np.int64)]))
