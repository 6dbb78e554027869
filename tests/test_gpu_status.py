"""Failure detection on the GPU without a fault: a bounded device wait that can
never complete gives up, the status word reports DCN_ERR_TIMEOUT through
dcn_check_status(), and the context keeps working."""
import numpy as np
import pytest
import torch

import oracle
import deformable_convolution_dcn_b200 as dcn
from deformable_convolution_dcn_b200 import inputs as gen

pytestmark = pytest.mark.gpu

ETIMEOUT = -4


def test_bounded_wait_gives_up_and_context_survives():
    lib = dcn._load()
    dcn.check_status()
    try:
        # about a millisecond of waiting on a barrier nothing arrives at
        assert lib.dcn_selftest_wait_timeout(2_000_000, None) == 0
        assert lib.dcn_check_status() == ETIMEOUT
        assert "bounded wait" in lib.dcn_last_error_string().decode()
    finally:
        lib.dcn_check_status()
    assert lib.dcn_check_status() == 0
    # the context is still usable: a small layer still matches the oracle
    w = gen.WORKLOADS["tiny"]
    d = gen.make_inputs(w)
    dd = {k: (None if v is None else v.cuda()) for k, v in d.items()}
    s = w.shape
    y = dcn.forward(dd["x"], dd["offset"], dd["mask"], dd["weight"], dd["bias"], s.stride, s.pad, s.dil)
    torch.cuda.synchronize()
    dcn.check_status()
    a = {k: gen.as_f64(v) for k, v in d.items()}
    ref = oracle.forward(a["x"], a["offset"], a["mask"], a["weight"], a["bias"], s.stride, s.pad, s.dil, s.G)
    assert np.max(np.abs(y.double().cpu().numpy() - ref) / (1 + np.abs(ref))) <= 1e-4
