"""dcn_forward_noalloc: the forward for callers that cannot allocate device memory.

Such callers (code whose device memory belongs to an allocator it cannot
reach, or code that must not call cudaMalloc while it runs because cudaMalloc
can synchronize the device) cannot provide the workspace that dcn_forward
takes. dcn_forward_noalloc keeps that scratch in one static device array
inside the library instead. These tests call it through the C ABI, on two
calls in a row with different inputs: each result must equal dcn_forward's bit
for bit (the same kernel, whose partial tiles are summed in a fixed order, so a
stale counter or partial left by the previous call would show), and must match
the float64 oracle (in full on the small shapes, at sampled output pixels on
the full conv4 layer). A shape needing more scratch than the array holds is
refused with a clear message.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import deformable_convolution_dcn_b200 as dcn
from deformable_convolution_dcn_b200 import inputs as gen

pytestmark = pytest.mark.gpu

DCN_ERR_WORKSPACE = -5
BF16_NORMWISE = 1e-2   # the tolerance of the bf16 parity tests


def _dev(d):
    return {k: (None if v is None else v.cuda()) for k, v in d.items()}


def _noalloc(lib, s, d, y):
    p = dcn._params(d["x"], d["weight"], d["offset"], s.stride, s.pad, s.dil, False)
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.dcn_forward_noalloc(ctypes.byref(p), ptr(d["x"]), ptr(d["offset"]), ptr(d["mask"]), ptr(d["weight"]),
                                   ptr(d["bias"]), ptr(y), stream)


def _oracle_rel(s, host, y, pixels=None):
    """Normwise error of y against the float64 oracle (at flat output pixels, or everywhere)."""
    a = {k: gen.as_f64(v) for k, v in host.items()}
    ref = oracle.forward(a["x"], a["offset"], a["mask"], a["weight"], a["bias"], s.stride, s.pad, s.dil, s.G,
                         pixels=pixels)
    got = y.double().cpu().numpy()
    if pixels is not None:
        got = got.reshape(-1, s.Cout)[pixels]
    return float(np.linalg.norm(got - ref) / np.linalg.norm(ref))


@pytest.mark.parametrize("shape", [
    gen.LayerShape(B=2, Cin=256, H=20, W=20, Cout=256),          # tiles shared by several CTAs
    gen.WORKLOADS["conv4"].shape,                                # the full conv4 layer
    gen.LayerShape(B=1, Cin=64, H=9, W=13, Cout=48, K=3, stride=2, pad=1, G=2),
], ids=["conv4_small", "conv4", "ragged_g2"])
def test_noalloc_matches_forward_twice(shape):
    lib = dcn._load()
    w = gen.Workload("noalloc", shape, "bf16", seed=31, bias=True)
    full = shape.P <= 1024
    pixels = None if full else np.unique(np.random.default_rng(5).choice(shape.P, 256, replace=False))
    for call, seed in enumerate((31, 32)):        # two calls in a row, different inputs
        host = gen.make_inputs(w, seed=seed)
        d = _dev(host)
        ref = dcn.forward(d["x"], d["offset"], d["mask"], d["weight"], d["bias"], shape.stride, shape.pad, shape.dil)
        y = torch.full_like(ref, float("nan"))
        rc = _noalloc(lib, shape, d, y)
        assert rc == 0, lib.dcn_last_error_string().decode()
        torch.cuda.synchronize()
        dcn.check_status()
        assert torch.isfinite(y.float()).all(), "call %d" % call
        assert torch.equal(y, ref), "call %d: differs from dcn_forward" % call
        rel = _oracle_rel(shape, host, y, pixels)
        assert rel <= BF16_NORMWISE, "call %d: normwise error %g against the oracle" % (call, rel)


def test_noalloc_refuses_shapes_beyond_its_scratch():
    lib = dcn._load()
    s = gen.WORKLOADS["conv5_d2g4"].shape          # 512 output channels: about 78 MB of partial tiles
    d = _dev(gen.make_inputs(gen.WORKLOADS["conv5_d2g4"]))
    p = dcn._params(d["x"], d["weight"], d["offset"], s.stride, s.pad, s.dil, False)
    if dcn.workspace_size(p, dcn.OP_FORWARD) <= 48 << 20:
        pytest.skip("this GPU's plan for the layer fits the static scratch")
    y = torch.empty((s.B, s.Ho, s.Wo, s.Cout), dtype=torch.bfloat16, device="cuda")
    assert _noalloc(lib, s, d, y) == DCN_ERR_WORKSPACE
    msg = lib.dcn_last_error_string().decode()
    assert "static array holds 50331648" in msg, msg
