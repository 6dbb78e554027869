"""Shapes printed on the pages (tests/golden/page_shapes.json) hold for the oracle."""
import json
import os

import numpy as np
import pytest

import oracle

CASES = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_shapes.json")))["cases"]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "K%d_G%d_%dx%d" % (c["K"], c["G"], c["H"], c["W"]))
def test_page_shapes_run_through_oracle(case):
    c = case
    r = np.random.default_rng(0)
    Ho, Wo = oracle.out_hw(c["H"], c["W"], c["K"], c["stride"], c["pad"], c["dil"])
    off_shape = (c["B"], 2 * c["G"] * c["K"] ** 2, Ho, Wo)
    assert list(off_shape) == c["offset_shape"]
    if "mask_shape" in c:
        assert [c["B"], c["G"] * c["K"] ** 2, Ho, Wo] == c["mask_shape"]
    if "weight_oihw" in c:
        assert [c["Cout"], c["Cin"], c["K"], c["K"]] == c["weight_oihw"]
    x = r.standard_normal((c["B"], c["H"], c["W"], c["Cin"]))
    w = r.standard_normal((c["Cout"], c["K"], c["K"], c["Cin"]))
    off = r.uniform(-1, 1, off_shape)
    mask = r.uniform(0, 1, (c["B"], c["G"] * c["K"] ** 2, Ho, Wo))
    y = oracle.forward(x, off, mask, w, None, c["stride"], c["pad"], c["dil"], c["G"])
    n, co, h, ww = c["y_nchw"]
    assert y.shape == (n, h, ww, co)
