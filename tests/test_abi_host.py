"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point that include/dcn.h declares, and rejects bad arguments with
the documented codes before anything reaches the device. No call here passes
valid device pointers, so nothing is launched."""
import ctypes

import pytest

import deformable_convolution_dcn_b200 as dcn

OK, EINVAL, EUNSUP, ECUDA, ETIMEOUT, EWS = 0, -1, -2, -3, -4, -5


@pytest.fixture(scope="module")
def lib():
    from deformable_convolution_dcn_b200 import build
    build.build()
    return dcn._load()


def P(**kw):
    d = dict(B=2, H=9, W=8, Cin=8, Cout=4, K=3, stride=1, pad=1, dil=1, G=2, dtype=0, flags=0)
    d.update(kw)
    return dcn.make_params(**d)


def test_exports_every_header_symbol(lib):
    names = dcn.header_symbols()
    assert {"dcn_forward", "dcn_backward_input", "dcn_backward_weight", "dcn_backward_offset_mask",
            "dcn_backward_data", "dcn_workspace_size", "dcn_last_error_string"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n
    assert lib.dcn_abi_version() == 2


def test_checked_build_exports_every_header_symbol():
    """The range-checked build (DCN_CHECKED) is the same library with checks
    compiled into its gather and scatter accesses: same entry points, same ABI."""
    import os
    from deformable_convolution_dcn_b200 import build
    path = build.build_checked()
    assert os.path.basename(path) == "libdcn_b200_checked.so"
    chk = ctypes.CDLL(path)
    for n in dcn.header_symbols():
        assert hasattr(chk, n), n
    chk.dcn_abi_version.restype = ctypes.c_int
    assert chk.dcn_abi_version() == 2


def test_library_override_is_restricted_to_package_builds():
    import subprocess
    import sys
    for bad in ("../evil.so", "/tmp/libdcn_b200.so", "libother.so"):
        r = subprocess.run([sys.executable, "-c", "import deformable_convolution_dcn_b200"], capture_output=True,
                           text=True, env={**__import__("os").environ, "DCN_B200_LIB": bad})
        assert r.returncode != 0 and "DCN_B200_LIB" in r.stderr, bad


@pytest.mark.parametrize("H,W,K,stride,pad,dil,expect", [
    (224, 224, 3, 1, 1, 1, (224, 224)), (200, 200, 3, 2, 1, 1, (100, 100)), (25, 25, 3, 1, 2, 2, (25, 25)),
    (50, 50, 3, 1, 1, 1, (50, 50)), (7, 5, 5, 2, 0, 1, (2, 1)), (1, 1, 3, 1, 1, 1, (1, 1)), (6, 6, 2, 1, 0, 1, (5, 5)),
])
def test_output_size(lib, H, W, K, stride, pad, dil, expect):
    assert dcn.output_size(P(H=H, W=W, K=K, stride=stride, pad=pad, dil=dil)) == expect


@pytest.mark.parametrize("bad,code", [
    (dict(B=0), EINVAL), (dict(H=-1), EINVAL), (dict(Cin=7, G=2), EINVAL), (dict(K=0), EINVAL),
    (dict(stride=0), EINVAL), (dict(pad=-1), EINVAL), (dict(dil=0), EINVAL), (dict(G=0), EINVAL),
    (dict(H=2, W=2, K=5, pad=0), EINVAL), (dict(dtype=7), EUNSUP),
    (dict(B=4096, H=1024, W=1024, Cin=8), EUNSUP),
])
def test_invalid_params_rejected(lib, bad, code):
    p = P(**bad)
    ho, wo = ctypes.c_int(), ctypes.c_int()
    assert lib.dcn_output_size(ctypes.byref(p), ctypes.byref(ho), ctypes.byref(wo)) == code
    assert lib.dcn_last_error_string().decode() != ""
    fake = ctypes.c_void_p(1 << 20)
    rc = lib.dcn_forward(ctypes.byref(p), fake, fake, None, fake, None, fake, None, 0, None)
    assert rc == code
    assert lib.dcn_workspace_size(ctypes.byref(p), 0) == 0
    assert dcn.forward_path(p) == "invalid"


def test_null_required_pointers(lib):
    p = P()
    f = ctypes.c_void_p(1 << 20)
    assert lib.dcn_forward(ctypes.byref(p), None, f, None, f, None, f, None, 0, None) == EINVAL
    assert "x is NULL" in lib.dcn_last_error_string().decode()
    assert lib.dcn_forward(ctypes.byref(p), f, None, None, f, None, f, None, 0, None) == EINVAL
    assert lib.dcn_forward(ctypes.byref(p), f, f, None, None, None, f, None, 0, None) == EINVAL
    assert lib.dcn_forward(ctypes.byref(p), f, f, None, f, None, None, None, 0, None) == EINVAL
    assert lib.dcn_backward_input(ctypes.byref(p), f, f, None, f, f, None, None, 0, None) == EINVAL
    assert lib.dcn_backward_offset_mask(ctypes.byref(p), f, f, None, f, f, None, None, None, 0, None) == EINVAL
    assert lib.dcn_backward_weight(ctypes.byref(p), f, f, None, f, None, None, None, 0, None) == EINVAL
    # grad_mask without a mask
    assert lib.dcn_backward_data(ctypes.byref(p), f, f, None, f, f, None, None, f, None, 0, None) == EINVAL
    assert lib.dcn_forward(None, f, f, None, f, None, f, None, 0, None) == EINVAL


def test_misaligned_pointers(lib):
    f = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 2)
    p32 = P(dtype=0)
    assert lib.dcn_forward(ctypes.byref(p32), odd, f, None, f, None, f, None, 0, None) == EUNSUP
    assert "aligned" in lib.dcn_last_error_string().decode()
    one = ctypes.c_void_p((1 << 20) + 1)
    p16 = P(dtype=1)
    assert lib.dcn_forward(ctypes.byref(p16), f, f, one, f, None, f, None, 0, None) == EUNSUP
    assert lib.dcn_backward_weight(ctypes.byref(p16), f, f, None, f, odd, None, None, 0, None) == EUNSUP


def test_predictor_arguments(lib):
    f = ctypes.c_void_p(1 << 20)
    p = P()
    n = lib.dcn_predict_workspace_size(ctypes.byref(p))
    # at least the zero offsets, the padded weights and the [P, 32] result
    P_ = 2 * 9 * 8
    assert n >= 4 * (P_ * 18 + 32 * 9 * 8 + P_ * 32)
    assert n % 256 == 0
    # Cout plays no part
    assert lib.dcn_predict_workspace_size(ctypes.byref(P(Cout=77))) == n
    assert lib.dcn_predict_workspace_size(ctypes.byref(P(B=0))) == 0
    assert lib.dcn_predict_offset_mask(ctypes.byref(P(B=0)), f, f, None, f, f, f, n, None) == EINVAL
    assert lib.dcn_predict_offset_mask(ctypes.byref(p), None, f, None, f, f, f, n, None) == EINVAL
    assert lib.dcn_predict_offset_mask(ctypes.byref(p), f, f, None, f, None, f, n, None) == EINVAL
    assert lib.dcn_predict_offset_mask(ctypes.byref(p), f, f, None, f, f, None, n, None) == EWS
    assert lib.dcn_predict_offset_mask(ctypes.byref(p), f, f, None, f, f, f, n - 1, None) == EWS
    assert str(n) in lib.dcn_last_error_string().decode()
    odd = ctypes.c_void_p((1 << 20) + 2)
    assert lib.dcn_predict_offset_mask(ctypes.byref(p), f, odd, None, f, f, f, n, None) == EUNSUP
    assert lib.dcn_predict_offset_mask(ctypes.byref(p), f, f, None, f, f, ctypes.c_void_p((1 << 20) + 128), n,
                                       None) == EUNSUP


def test_predictor_tensor_core_path_needs_no_workspace(lib):
    f = ctypes.c_void_p(1 << 20)
    p16 = P(dtype=1, Cin=64, G=1)
    assert lib.dcn_predict_workspace_size(ctypes.byref(p16)) == 0
    # stride 2 and float32 layers take the forward-kernel path, which does
    assert lib.dcn_predict_workspace_size(ctypes.byref(P(dtype=1, Cin=64, G=1, stride=2))) > 0
    assert lib.dcn_predict_workspace_size(ctypes.byref(P(dtype=0, Cin=64, G=1))) > 0
    # its tensor maps need 16-byte aligned x and w_pred
    odd = ctypes.c_void_p((1 << 20) + 2)
    assert lib.dcn_predict_offset_mask(ctypes.byref(p16), odd, f, None, f, f, None, 0, None) == EUNSUP
    assert "16-byte" in lib.dcn_last_error_string().decode()
    assert lib.dcn_predict_offset_mask(ctypes.byref(p16), f, odd, None, f, f, None, 0, None) == EUNSUP


def test_roi_pool_arguments(lib):
    f = ctypes.c_void_p(1 << 20)

    def RP(**kw):
        d = dict(B=2, H=8, W=9, C=16, R=5, k=3, gamma=0.5, dtype=0, flags=0)
        d.update(kw)
        return dcn.RoiParams(d["B"], d["H"], d["W"], d["C"], d["R"], d["k"], d["gamma"], d["dtype"], d["flags"])

    fwd = lambda p, *a: lib.dcn_droi_pool_forward(ctypes.byref(p), *a, None)
    bwd = lambda p, *a: lib.dcn_droi_pool_backward(ctypes.byref(p), *a, None)
    for bad, code in ((dict(k=0), EINVAL), (dict(k=65), EINVAL), (dict(R=-1), EINVAL), (dict(C=0), EINVAL),
                      (dict(B=0), EINVAL), (dict(dtype=9), EUNSUP), (dict(gamma=float("nan")), EINVAL),
                      (dict(gamma=float("inf")), EINVAL), (dict(B=1024, H=1024, W=1024, C=8), EUNSUP)):
        assert fwd(RP(**bad), f, f, None, None, f) == code, bad
        assert lib.dcn_last_error_string().decode() != ""
    assert fwd(RP(), None, f, None, None, f) == EINVAL
    assert "x is NULL" in lib.dcn_last_error_string().decode()
    assert fwd(RP(), f, None, None, None, f) == EINVAL
    assert fwd(RP(), f, f, None, None, None) == EINVAL
    assert fwd(RP(), f, ctypes.c_void_p((1 << 20) + 2), None, None, f) == EUNSUP
    assert fwd(RP(dtype=1), f, f, ctypes.c_void_p((1 << 20) + 1), None, f) == EUNSUP
    # no RoIs: nothing to do, nothing enqueued
    assert fwd(RP(R=0), f, None, None, None, None) == OK
    # gradients of absent inputs, and the required grad_x
    assert bwd(RP(), f, f, None, None, f, f, f, None) == EINVAL
    assert "grad_offset needs offset" in lib.dcn_last_error_string().decode()
    assert bwd(RP(), f, f, f, None, f, f, None, f) == EINVAL
    assert "grad_mask needs mask" in lib.dcn_last_error_string().decode()
    assert bwd(RP(), f, f, f, f, f, None, None, None) == EINVAL
    assert bwd(RP(), f, f, f, f, None, f, None, None) == EINVAL


def test_selftest_rejects_out_of_range_limits(lib):
    assert lib.dcn_selftest_wait_timeout(10, None) == EINVAL
    assert lib.dcn_selftest_wait_timeout(5_000_000_000, None) == EINVAL
    assert "limit_cycles" in lib.dcn_last_error_string().decode()


def test_python_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import importlib
    monkeypatch.setattr(dcn, "_lib", None)
    monkeypatch.setattr(dcn, "_LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="not built"):
        dcn._load()


F32, BF16 = 0, 1


@pytest.mark.parametrize("kw,flags,expect", [
    # float32 RGB-like layers: the split-tf32 tensor-core kernel
    (dict(B=1, H=224, W=224, Cin=3, Cout=64, G=1, dtype=F32), 0, "tcgen05_tf32_split"),
    (dict(B=1, H=224, W=224, Cin=3, Cout=64, G=1, dtype=F32), dcn.DCN_FLAG_NO_TF32, "f32_small_channels"),
    (dict(B=1, H=224, W=224, Cin=3, Cout=64, G=1, dtype=F32), dcn.DCN_FLAG_GENERIC, "generic"),
    (dict(B=1, H=20, W=21, Cin=1, Cout=256, G=1, dtype=F32), 0, "tcgen05_tf32_split"),
    # outside the split-tf32 kernel's shapes: Cin > 3, K*K > 9, groups, Cout not a multiple of 32
    (dict(B=1, H=31, W=17, Cin=4, Cout=64, G=1, dtype=F32), 0, "f32_small_channels"),
    (dict(B=2, H=9, W=12, Cin=1, Cout=32, K=5, pad=2, G=1, dtype=F32), 0, "f32_small_channels"),
    (dict(B=2, H=6, W=9, Cin=2, Cout=32, G=2, dtype=F32), 0, "f32_small_channels"),
    (dict(B=1, H=16, W=16, Cin=3, Cout=48, G=1, dtype=F32), 0, "generic"),
    (dict(B=1, H=16, W=16, Cin=16, Cout=64, G=1, dtype=F32), 0, "generic"),
    # bfloat16: the tcgen05 gather kernel for channel counts in multiples of 8
    (dict(B=8, H=50, W=50, Cin=256, Cout=256, G=1, dtype=BF16), 0, "tcgen05_gather_tmem"),
    # 7x7: records held one kernel row (seven taps) at a time
    (dict(B=1, H=11, W=9, Cin=16, Cout=24, K=7, pad=3, G=1, dtype=BF16), 0, "tcgen05_gather_tmem"),
    (dict(B=1, H=11, W=9, Cin=16, Cout=264, K=7, pad=3, G=1, dtype=BF16), 0, "generic"),
    (dict(B=8, H=50, W=50, Cin=256, Cout=256, G=1, dtype=BF16), dcn.DCN_FLAG_GENERIC, "generic"),
    (dict(B=8, H=25, W=25, Cin=512, Cout=512, G=4, pad=2, dil=2, dtype=BF16), 0, "tcgen05_gather"),
    (dict(B=1, H=9, W=9, Cin=12, Cout=16, G=1, dtype=BF16), 0, "generic"),
])
def test_forward_dispatch(lib, kw, flags, expect):
    """Which forward kernel a layer gets, decided on the host before any launch."""
    assert dcn.forward_path(P(flags=flags, **kw)) == expect
