"""GPU parity of the offset/mask predictor (a plain convolution with 3*G*K*K
outputs, the first 2*G*K*K the offsets and the rest the sigmoid masks: notes,
DCNv2 section 3.2) against the float64 oracle, compared in full."""
import numpy as np
import pytest
import torch

import oracle
import deformable_convolution_dcn_b200 as dcn
from deformable_convolution_dcn_b200 import inputs as gen
from parity import assert_close, f64, to_dev

pytestmark = pytest.mark.gpu

S = gen.LayerShape

SHAPES = [
    # RGB stem-like (float32: the split-tf32 kernel, 27 outputs padded to 32)
    (S(B=1, Cin=3, H=24, W=24, Cout=1), "f32"),
    (S(B=2, Cin=3, H=17, W=13, Cout=1, stride=2), "f32"),
    # float32 CUDA-core path, ragged sizes, two offset groups, stride 2
    (S(B=2, Cin=16, H=13, W=11, Cout=1, stride=2, G=2), "f32"),
    (S(B=1, Cin=12, H=9, W=10, Cout=1, K=5, pad=2, G=3), "f32"),
    (S(B=1, Cin=8, H=7, W=6, Cout=1, K=1, pad=0), "f32"),
    # bfloat16 tensor-core path
    (S(B=2, Cin=64, H=13, W=11, Cout=1), "bf16"),
    (S(B=1, Cin=256, H=12, W=10, Cout=1, pad=2, dil=2, G=4), "bf16"),
    (S(B=1, Cin=48, H=9, W=21, Cout=1, K=5, pad=2, G=2), "bf16"),
    (S(B=2, Cin=16, H=8, W=8, Cout=1, K=1, pad=0), "bf16"),
    (S(B=1, Cin=128, H=17, W=9, Cout=1, stride=2), "bf16"),
    # bfloat16 stride 1: the implicit-GEMM kernel (ragged slabs and tiles, no padding, dilation, wide rows)
    (S(B=3, Cin=136, H=20, W=30, Cout=1), "bf16"),
    (S(B=1, Cin=8, H=40, W=100, Cout=1), "bf16"),
    (S(B=2, Cin=64, H=9, W=9, Cout=1, pad=0), "bf16"),
    (S(B=1, Cin=32, H=11, W=13, Cout=1, pad=1, dil=2), "bf16"),
    (S(B=2, Cin=24, H=6, W=7, Cout=1, K=1, pad=0, G=2), "bf16"),
]


def _ids(c):
    s, dt = c
    return "%s-B%dC%dH%dW%dK%ds%dd%dG%d" % (dt, s.B, s.Cin, s.H, s.W, s.K, s.stride, s.dil, s.G)


def _run(s, d, generic=False):
    off, m = dcn.predict_offset_mask(d["x"], d["w_pred"], d["b_pred"], s.K, s.stride, s.pad, s.dil, s.G,
                                     generic=generic)
    torch.cuda.synchronize()
    dcn.check_status()
    return off.float().cpu().numpy(), m.float().cpu().numpy()


def _ref(s, a):
    return oracle.predict_offset_mask(a["x"], a["w_pred"], a["b_pred"], s.K, s.stride, s.pad, s.dil, s.G)


@pytest.mark.parametrize("case", SHAPES, ids=[_ids(c) for c in SHAPES])
@pytest.mark.parametrize("bias", [True, False], ids=["bias", "nobias"])
def test_predictor_matches_oracle(case, bias):
    s, dt = case
    d = gen.predictor_inputs(11, s, dt, bias=bias)
    off, m = _run(s, to_dev(d))
    roff, rm = _ref(s, f64(d))
    assert_close(off, roff, dt, "offset")
    assert_close(m, rm, dt, "mask")
    assert np.all((m >= 0) & (m <= 1))


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_predictor_generic_path_agrees(dt):
    s = S(B=2, Cin=64, H=13, W=11, Cout=1, G=2)
    d = gen.predictor_inputs(12, s, dt)
    roff, rm = _ref(s, f64(d))
    off, m = _run(s, to_dev(d), generic=True)
    assert_close(off, roff, dt, "offset")
    assert_close(m, rm, dt, "mask")


def test_predictor_conv4_full_size():
    """The predictor of the ResNet-50 conv4 layer (B8, 256 channels, 50x50,
    3x3, bfloat16), compared in full."""
    s = gen.WORKLOADS["conv4"].shape
    d = gen.predictor_inputs(13, s, "bf16")
    off, m = _run(s, to_dev(d))
    roff, rm = _ref(s, f64(d))
    assert_close(off, roff, "bf16", "offset")
    assert_close(m, rm, "bf16", "mask")


def test_predictor_zero_weights_give_bias_and_half():
    """The DCNv2 start: zero predictor weights and bias give zero offsets and
    masks of exactly 0.5."""
    s = S(B=1, Cin=32, H=10, W=10, Cout=1)
    d = gen.predictor_inputs(14, s, "bf16", bias=False)
    d["w_pred"].zero_()
    off, m = _run(s, to_dev(d))
    assert np.all(off == 0.0)
    assert np.all(m == 0.5)


def test_predictor_feeds_the_layer():
    """Predictor then layer, both on the GPU, against the oracle's predictor
    then the oracle's layer (float32)."""
    s = S(B=1, Cin=16, H=11, W=12, Cout=24, G=2)
    d = gen.predictor_inputs(15, s, "f32")
    g = torch.Generator().manual_seed(16)
    w = (torch.randn((s.Cout, s.K, s.K, s.Cin), generator=g) * 0.2)
    dd = to_dev(d)
    off, m = dcn.predict_offset_mask(dd["x"], dd["w_pred"], dd["b_pred"], s.K, s.stride, s.pad, s.dil, s.G)
    y = dcn.forward(dd["x"], off, m, w.cuda(), None, s.stride, s.pad, s.dil)
    torch.cuda.synchronize()
    dcn.check_status()
    a = f64(d)
    roff, rm = _ref(s, a)
    ry = oracle.forward(a["x"], roff, rm, w.double().numpy(), None, s.stride, s.pad, s.dil, s.G)
    assert_close(y.cpu().numpy(), ry, "f32", "y")
