"""GPU parity of (modulated) deformable RoI pooling against the float64 oracle,
forward and backward, compared in full."""
import numpy as np
import pytest
import torch

import oracle
import deformable_convolution_dcn_b200 as dcn
from deformable_convolution_dcn_b200 import inputs as gen
from parity import assert_close

pytestmark = pytest.mark.gpu

# gamma dyadic and offsets on a 1/64 grid: every sample position is exact in
# float32 and float64, so both sides take the same neighbours
CASES = [
    # B, H, W, C, R, k, gamma, offsets, mask, max_side
    (2, 20, 24, 32, 40, 3, 0.5, True, True, None),
    (1, 13, 9, 8, 17, 7, 1.0, True, False, None),
    (2, 16, 16, 64, 25, 2, 0.125, False, False, None),
    (1, 11, 14, 5, 30, 4, 0.25, True, True, 3.0),
    (3, 8, 10, 256, 12, 7, 0.125, True, True, None),
]


def _f64(d):
    return {k: gen.as_f64(v) for k, v in d.items()}


def _ids(c):
    return "B%dH%dW%dC%dR%dk%d%s%s" % (c[0], c[1], c[2], c[3], c[4], c[5], "off" if c[7] else "",
                                         "mask" if c[8] else "")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("case", CASES, ids=[_ids(c) for c in CASES])
def test_droi_pool_matches_oracle(case, dtype):
    B, H, W, C, R, k, gamma, offs, mask, side = case
    d = gen.roi_inputs(31, B, H, W, C, R, k, dtype, offsets=offs, mask=mask, max_side=side)
    dd = {n: (None if v is None else v.cuda()) for n, v in d.items()}
    y = dcn.droi_pool_forward(dd["x"], dd["rois"], dd["offset"], dd["mask"], k, gamma)
    gx, goff, gm = dcn.droi_pool_backward(dd["x"], dd["rois"], dd["offset"], dd["mask"], dd["grad_y"], k, gamma)
    torch.cuda.synchronize()
    dcn.check_status()
    a = _f64(d)
    ry = oracle.droi_pool_forward(a["x"], a["rois"], a["offset"], a["mask"], k, gamma)
    rgx, rgoff, rgm = oracle.droi_pool_backward(a["x"], a["rois"], a["offset"], a["mask"], a["grad_y"], k, gamma)
    assert_close(y.float().cpu().numpy(), ry, dtype, "y")
    assert_close(gx.cpu().numpy(), rgx, dtype, "grad_x")
    if offs:
        assert_close(goff.cpu().numpy(), rgoff, dtype, "grad_offset")
    else:
        assert goff is None
    if mask:
        assert_close(gm.cpu().numpy(), rgm, dtype, "grad_mask")
    else:
        assert gm is None


def test_droi_pool_degenerate_rois():
    """Zero-size RoIs and RoIs wholly outside the map pool to zeros; a batch
    index outside [0, B) gives zeros and no gradient."""
    x = torch.randn((2, 6, 7, 16), device="cuda")
    rois = torch.tensor([[0, 2, 2, 2, 5], [1, 20, 20, 30, 30], [0, -9, -9, -3, -2], [5, 1, 1, 4, 4],
                         [-1, 1, 1, 4, 4], [1, 1, 1, 4, 4]], dtype=torch.float32, device="cuda")
    y = dcn.droi_pool_forward(x, rois, None, None, 3)
    gy = torch.ones((6, 3, 3, 16), device="cuda")
    gx, _, _ = dcn.droi_pool_backward(x, rois, None, None, gy, 3)
    torch.cuda.synchronize()
    assert torch.all(y[:5] == 0)
    assert torch.any(y[5] != 0)
    # only the last RoI (batch 1, 3 x 3 pixels) receives gradient: each of its pixels once per bin it is in
    assert torch.all(gx[0] == 0)
    assert float(gx[1].sum()) == pytest.approx(16 * 9.0, rel=1e-6)


def test_droi_pool_no_rois():
    x = torch.randn((1, 5, 5, 8), device="cuda")
    rois = torch.zeros((0, 5), dtype=torch.float32, device="cuda")
    y = dcn.droi_pool_forward(x, rois, None, None, 2)
    gx, _, _ = dcn.droi_pool_backward(x, rois, None, None, torch.zeros((0, 2, 2, 8), device="cuda"), 2)
    torch.cuda.synchronize()
    assert y.shape == (0, 2, 2, 8) and torch.all(gx == 0)
