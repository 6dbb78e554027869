"""Failure detection on the GPU without a fault: a bounded device wait that can
never complete gives up, the status word reports DCN_ERR_TIMEOUT through
dcn_check_status(stream), and the context keeps working; the check waits for
its own stream only."""
import ctypes
import time

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
        assert lib.dcn_check_status(None) == ETIMEOUT
        assert "bounded wait" in lib.dcn_last_error_string().decode()
    finally:
        lib.dcn_check_status(None)
    assert lib.dcn_check_status(None) == 0
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


def test_timeout_on_a_side_stream_is_reported_through_that_stream():
    lib = dcn._load()
    dcn.check_status()
    side = torch.cuda.Stream()
    h = ctypes.c_void_p(side.cuda_stream)
    assert lib.dcn_selftest_wait_timeout(2_000_000, h) == 0
    assert lib.dcn_check_status(h) == ETIMEOUT
    assert lib.dcn_check_status(h) == 0  # taken and cleared
    dcn.check_status(side)


def test_check_status_waits_for_its_stream_only():
    lib = dcn._load()
    busy, quiet = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(busy):
        torch.cuda._sleep(2_000_000_000)  # about a second of device time on the other stream
    t0 = time.perf_counter()
    assert lib.dcn_check_status(ctypes.c_void_p(quiet.cuda_stream)) == 0
    dt = time.perf_counter() - t0
    busy.synchronize()
    assert dt < 0.5, "dcn_check_status waited %.3f s for another stream" % dt
