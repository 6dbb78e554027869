"""GPU parity: the CUDA library (through the C ABI) against the float64 oracle.

Small layers are compared in full, element by element; the full-size layer
shapes are compared at sampled output pixels / gradient entries that the
oracle computes one by one, plus identities that hold at any size.
"""
import numpy as np
import pytest
import torch

import oracle
import deformable_convolution_dcn_b200 as dcn
from deformable_convolution_dcn_b200 import inputs as gen
from parity import assert_close, f64, run_backward, run_forward, sample_pixels, to_dev

pytestmark = pytest.mark.gpu


def _oracle_forward(s, a, pixels=None):
    return oracle.forward(a["x"], a["offset"], a["mask"], a["weight"], a["bias"], s.stride, s.pad, s.dil, s.G,
                          pixels=pixels)


def _oracle_backward(s, a):
    return oracle.backward(a["x"], a["offset"], a["mask"], a["weight"], a["grad_y"], s.stride, s.pad, s.dil, s.G)


def _cpu(t):
    return None if t is None else t.float().cpu().numpy()


# ------------------------------------------------------------ small, in full --

@pytest.mark.parametrize("generic", [False, True], ids=["default", "generic"])
def test_tiny_forward_backward(generic):
    w = gen.WORKLOADS["tiny"]
    s = w.shape
    d = gen.make_inputs(w)
    a = f64(d)
    dd = to_dev(d)
    y = run_forward(s, dd, generic)
    assert_close(_cpu(y), _oracle_forward(s, a), "f32", "y")
    g = run_backward(s, dd, generic)
    ref = _oracle_backward(s, a)
    for k in ("grad_x", "grad_offset", "grad_mask", "grad_weight", "grad_bias"):
        assert_close(_cpu(g[k]), ref[k], "f32", k)


CASES = list(range(24))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("seed", CASES)
def test_random_small_layers(seed, dtype):
    s, d = gen.random_case(seed, dtype, with_mask=(seed % 5 != 4), with_bias=(seed % 3 != 2))
    a = f64(d)
    dd = to_dev(d)
    y = run_forward(s, dd)
    assert_close(_cpu(y), _oracle_forward(s, a), dtype, "y %s" % (s,))
    g = run_backward(s, dd)
    ref = _oracle_backward(s, a)
    for k in ("grad_x", "grad_offset", "grad_mask", "grad_weight", "grad_bias"):
        if ref[k] is None:
            assert g[k] is None
            continue
        assert_close(_cpu(g[k]), ref[k], dtype if dtype == "f32" else "bf16", "%s %s" % (k, s))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [
    gen.LayerShape(B=2, Cin=64, H=13, W=11, Cout=40, K=3, stride=1, pad=1),
    gen.LayerShape(B=1, Cin=128, H=17, W=9, Cout=136, K=3, stride=2, pad=1),
    gen.LayerShape(B=3, Cin=96, H=10, W=10, Cout=64, K=3, stride=1, pad=2, dil=2, G=4),
    gen.LayerShape(B=1, Cin=48, H=9, W=21, Cout=24, K=5, stride=1, pad=2, G=2),
    gen.LayerShape(B=2, Cin=256, H=12, W=12, Cout=256, K=3, stride=1, pad=1),
    gen.LayerShape(B=1, Cin=512, H=7, W=7, Cout=512, K=3, stride=1, pad=2, dil=2, G=4),
], ids=lambda s: "B%dC%dx%dH%dW%dK%ds%dd%dG%d" % (s.B, s.Cin, s.Cout, s.H, s.W, s.K, s.stride, s.dil, s.G))
def test_medium_layers_span_tiles(shape, dtype):
    """Several tiles and a ragged tail in every dimension; compared in full."""
    w = gen.Workload("medium", shape, dtype, seed=7, offset_dist="normal1.5_edges", bias=True, backward=True)
    d = gen.make_inputs(w)
    a = f64(d)
    dd = to_dev(d)
    y = run_forward(shape, dd)
    assert_close(_cpu(y), _oracle_forward(shape, a), dtype, "y")
    g = run_backward(shape, dd)
    ref = _oracle_backward(shape, a)
    for k in ("grad_x", "grad_offset", "grad_mask", "grad_weight", "grad_bias"):
        assert_close(_cpu(g[k]), ref[k], dtype, k)


# --------------------------------------------------------------- edge cases --

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_samples_all_outside_give_bias(dtype):
    s, d = gen.random_case(3, dtype, Cin=16, Cout=24, H=9, W=9, K=3, G=1)
    d["offset"] = torch.full_like(d["offset"], 100.0)
    dd = to_dev(d)
    y = run_forward(s, dd)
    expect = d["bias"].float().numpy()
    assert np.array_equal(_cpu(y), np.broadcast_to(expect, y.shape))
    g = run_backward(s, dd)
    assert float(g["grad_x"].abs().max()) == 0.0
    assert float(g["grad_offset"].abs().max()) == 0.0
    assert float(g["grad_weight"].abs().max()) == 0.0


@pytest.mark.parametrize("spread", [0.3, 2.5], ids=["converging", "crowded"])
def test_backward_converging_samples(spread):
    """Offsets that pull every sample of a tap towards one point of the map: the
    input pixels there receive far more bilinear corners than the per-pixel
    lists of the transposed grad_x pass hold (spread 0.3: hundreds each, all
    left to the atomic scatter; 2.5: tens, partly kept). Full backward against
    the oracle, element by element."""
    s, d = gen.random_case(21, "bf16", B=2, Cin=64, Cout=64, H=11, W=13, K=3, stride=1, pad=1, dil=1, G=1)
    g = torch.Generator().manual_seed(22)
    ho = torch.arange(s.Ho, dtype=torch.float32).view(1, 1, s.Ho, 1)
    wo = torch.arange(s.Wo, dtype=torch.float32).view(1, 1, 1, s.Wo)
    off = torch.empty((s.B, 2 * s.K * s.K, s.Ho, s.Wo))
    for tap in range(s.K * s.K):
        i, j = divmod(tap, s.K)
        # sample row = ho - pad + i + dy lands near row 5.3, column near 6.6
        off[:, 2 * tap] = (5.3 - (ho - s.pad + i) + spread * torch.randn((s.B, 1, s.Ho, s.Wo), generator=g))[:, 0]
        off[:, 2 * tap + 1] = (6.6 - (wo - s.pad + j) + spread * torch.randn((s.B, 1, s.Ho, s.Wo), generator=g))[:, 0]
    d["offset"] = off.to(d["offset"].dtype)
    a = f64(d)
    g_ = run_backward(s, to_dev(d))
    ref = _oracle_backward(s, a)
    for k in ("grad_x", "grad_offset", "grad_mask", "grad_weight", "grad_bias"):
        assert_close(_cpu(g_[k]), ref[k], "bf16", k)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_mask_zero_gives_bias(dtype):
    s, d = gen.random_case(4, dtype, Cin=32, Cout=16, H=8, W=10)
    d["mask"] = torch.zeros_like(d["mask"])
    y = run_forward(s, to_dev(d))
    assert np.array_equal(_cpu(y), np.broadcast_to(d["bias"].float().numpy(), y.shape))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_zero_offsets_match_conv2d(dtype):
    """Zero offsets and unit mask: the layer is torch's own conv2d (float64 on the CPU)."""
    s, d = gen.random_case(5, dtype, Cin=64, Cout=32, H=11, W=13, K=3, stride=1, pad=1, dil=1, G=1)
    d["offset"] = torch.zeros_like(d["offset"])
    d["mask"] = torch.ones_like(d["mask"])
    y = run_forward(s, to_dev(d))
    a = f64(d)
    ref = torch.nn.functional.conv2d(torch.from_numpy(a["x"]).permute(0, 3, 1, 2),
                                     torch.from_numpy(a["weight"]).permute(0, 3, 1, 2), torch.from_numpy(a["bias"]),
                                     stride=s.stride, padding=s.pad, dilation=s.dil).permute(0, 2, 3, 1).numpy()
    assert_close(_cpu(y), ref, dtype, "y")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_single_output_pixel_and_one_channel(dtype):
    for kw in (dict(B=1, Cin=8, Cout=1, H=1, W=1, K=3, pad=1), dict(B=1, Cin=8, Cout=3, H=3, W=3, K=3, pad=0),
               dict(B=2, Cin=8, Cout=8, H=2, W=9, K=1, pad=0)):
        s, d = gen.random_case(6, dtype, **kw)
        a = f64(d)
        dd = to_dev(d)
        assert_close(_cpu(run_forward(s, dd)), _oracle_forward(s, a), dtype, "y %s" % (s,))
        g = run_backward(s, dd)
        ref = _oracle_backward(s, a)
        for k in ("grad_x", "grad_offset", "grad_mask", "grad_weight", "grad_bias"):
            assert_close(_cpu(g[k]), ref[k], dtype, k)


def test_repeated_calls_identical():
    """The same call twice gives bit-identical forward outputs."""
    w = gen.WORKLOADS["conv4"]
    s = gen.LayerShape(B=2, Cin=256, H=20, W=20, Cout=256)
    dd = to_dev(gen.make_inputs(w, shape=s))
    y1 = run_forward(s, dd)
    y2 = run_forward(s, dd)
    assert torch.equal(y1, y2)


# ---------------------------------------------------------- full-size shapes --

@pytest.mark.parametrize("name", ["stem", "conv4", "conv3_s2", "conv5_d2g4", "conv4_v1", "conv4_k5"])
def test_full_size_forward_sampled(name):
    w = gen.WORKLOADS[name]
    s = w.shape
    d = gen.make_inputs(w)
    a = f64(d)
    y = run_forward(s, to_dev(d))
    pix = sample_pixels(s, 96, seed=11)
    ref = _oracle_forward(s, a, pixels=pix)
    got = _cpu(y).reshape(s.P, s.Cout)[pix]
    assert_close(got, ref, w.dtype, name)


def test_full_size_forward_generic_agrees():
    """The generic kernel and the default path agree on the conv4 layer."""
    w = gen.WORKLOADS["conv4"]
    s = w.shape
    dd = to_dev(gen.make_inputs(w))
    y = run_forward(s, dd).float()
    yg = run_forward(s, dd, generic=True).float()
    rel = float((y - yg).norm() / yg.norm())
    assert rel <= 1e-2, rel


def test_full_size_backward_sampled():
    w = gen.WORKLOADS["conv4_bwd"]
    s = w.shape
    d = gen.make_inputs(w)
    a = f64(d)
    dd = to_dev(d)
    g = run_backward(s, dd)
    pix = sample_pixels(s, 48, seed=12)
    goff, gm = oracle.grad_offset_mask_at(a["x"], a["offset"], a["mask"], a["weight"], a["grad_y"], pix, s.stride,
                                          s.pad, s.dil, s.G)
    got_off = _cpu(g["grad_offset"]).transpose(0, 2, 3, 1).reshape(s.P, -1)[pix]
    got_m = _cpu(g["grad_mask"]).transpose(0, 2, 3, 1).reshape(s.P, -1)[pix]
    assert_close(got_off, goff, "bf16", "grad_offset")
    assert_close(got_m, gm, "bf16", "grad_mask")
    r = np.random.default_rng(13)
    went = r.choice(s.Cout * s.K * s.K * s.Cin, 64, replace=False)
    gw_ref = oracle.grad_weight_at(a["x"], a["offset"], a["mask"], a["grad_y"], a["weight"].shape, went, s.stride,
                                   s.pad, s.dil, s.G)
    assert_close(_cpu(g["grad_weight"]).reshape(-1)[went], gw_ref, "bf16", "grad_weight")
    xent = r.choice(s.B * s.H * s.W * s.Cin, 64, replace=False)
    gx_ref = oracle.grad_x_at(a["x"].shape, a["offset"], a["mask"], a["weight"], a["grad_y"], xent, s.stride, s.pad,
                              s.dil, s.G)
    assert_close(_cpu(g["grad_x"]).reshape(-1)[xent], gx_ref, "bf16", "grad_x")
    assert_close(_cpu(g["grad_bias"]), a["grad_y"].sum(axis=(0, 1, 2)), "bf16", "grad_bias")
    # identity at full size: <grad_y, y - bias> = <grad_x, x> = <grad_w, w> = <grad_mask, mask>
    y = run_forward(s, dd).double()
    gy = dd["grad_y"].double()
    lhs = float((gy * y).sum())
    for gname, prim in (("grad_x", "x"), ("grad_weight", "weight"), ("grad_mask", "mask")):
        rhs = float((g[gname].double() * dd[prim].double()).sum())
        assert abs(lhs - rhs) <= 2e-2 * abs(lhs), (gname, lhs, rhs)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape,mask", [
    (gen.LayerShape(B=1, Cin=16, H=11, W=9, Cout=24, K=7, pad=3), True),
    (gen.LayerShape(B=2, Cin=32, H=9, W=14, Cout=16, K=7, pad=3, dil=1, G=2), False),
    (gen.LayerShape(B=1, Cin=8, H=16, W=10, Cout=8, K=7, stride=2, pad=6, dil=2), True),
    # two 64-channel slices, six tiles split over many CTAs: stream-K segments start inside a tap row
    (gen.LayerShape(B=2, Cin=128, H=20, W=18, Cout=64, K=7, pad=3), True),
], ids=["k7", "k7_g2_v1", "k7_s2_d2", "k7_c128"])
def test_seven_by_seven_layers(shape, mask, dtype):
    """K = 7 (49 taps, 98 offset channels per group), DCNv2 and DCNv1, forward and backward in full;
    the bf16 forward runs on the TMEM-operand tensor-core kernel."""
    w = gen.Workload("k7", shape, dtype, seed=17, offset_dist="uniform2.5",
                     mask_dist="uniform" if mask else "none", bias=True, backward=True)
    d = gen.make_inputs(w)
    if dtype == "bf16":
        p = dcn._params(d["x"], d["weight"], d["offset"], shape.stride, shape.pad, shape.dil, False)
        assert dcn.forward_path(p) == "tcgen05_gather_tmem"
    a = f64(d)
    dd = to_dev(d)
    assert_close(_cpu(run_forward(shape, dd)), _oracle_forward(shape, a), dtype, "y")
    g = run_backward(shape, dd)
    ref = _oracle_backward(shape, a)
    for k in ("grad_x", "grad_offset", "grad_mask", "grad_weight", "grad_bias"):
        if ref[k] is None:
            assert g[k] is None
            continue
        assert_close(_cpu(g[k]), ref[k], dtype, k)


def test_full_size_v1_backward_sampled():
    """DCNv1 (no mask) backward on the conv4 layer at sampled entries."""
    w = gen.WORKLOADS["conv4_v1"]
    s = w.shape
    d = gen.make_inputs(w)
    g0 = torch.Generator().manual_seed(21)
    d["grad_y"] = torch.randn((s.B, s.Ho, s.Wo, s.Cout), generator=g0).to(torch.bfloat16)
    a = f64(d)
    g = run_backward(s, to_dev(d))
    assert g["grad_mask"] is None
    pix = sample_pixels(s, 32, seed=22)
    goff, _ = oracle.grad_offset_mask_at(a["x"], a["offset"], None, a["weight"], a["grad_y"], pix, s.stride, s.pad,
                                         s.dil, s.G)
    got_off = _cpu(g["grad_offset"]).transpose(0, 2, 3, 1).reshape(s.P, -1)[pix]
    assert_close(got_off, goff, "bf16", "grad_offset")
    r = np.random.default_rng(23)
    went = r.choice(s.Cout * s.K * s.K * s.Cin, 48, replace=False)
    gw_ref = oracle.grad_weight_at(a["x"], a["offset"], None, a["grad_y"], a["weight"].shape, went, s.stride, s.pad,
                                   s.dil, s.G)
    assert_close(_cpu(g["grad_weight"]).reshape(-1)[went], gw_ref, "bf16", "grad_weight")
    xent = r.choice(s.B * s.H * s.W * s.Cin, 48, replace=False)
    gx_ref = oracle.grad_x_at(a["x"].shape, a["offset"], None, a["weight"], a["grad_y"], xent, s.stride, s.pad,
                              s.dil, s.G)
    assert_close(_cpu(g["grad_x"]).reshape(-1)[xent], gx_ref, "bf16", "grad_x")


def _tf32_split_applies(s):
    """The float32 tensor-core kernel takes Cin <= 3, one group, K*K <= 9, Cout a multiple of 32 up to 256."""
    return s.Cin <= 3 and s.G == 1 and s.K * s.K <= 9 and s.Cout % 32 == 0 and 32 <= s.Cout <= 256


@pytest.mark.parametrize("kernel", ["default", "cuda_cores"])
@pytest.mark.parametrize("shape,mask", [
    (gen.LayerShape(B=1, Cin=3, H=23, W=19, Cout=64, K=3, stride=1, pad=1), True),
    (gen.LayerShape(B=2, Cin=3, H=17, W=30, Cout=128, K=3, stride=2, pad=1), True),
    (gen.LayerShape(B=1, Cin=2, H=13, W=11, Cout=32, K=3, stride=1, pad=2, dil=2), True),
    (gen.LayerShape(B=1, Cin=1, H=20, W=21, Cout=256, K=3, stride=1, pad=0), True),
    (gen.LayerShape(B=1, Cin=3, H=9, W=40, Cout=128, K=1, stride=1, pad=0), False),
    (gen.LayerShape(B=2, Cin=1, H=9, W=12, Cout=32, K=5, stride=2, pad=2), True),
    (gen.LayerShape(B=1, Cin=8, H=10, W=7, Cout=128, K=3, stride=1, pad=2, dil=2, G=2), True),
    (gen.LayerShape(B=2, Cin=2, H=6, W=9, Cout=16, K=3, stride=1, pad=1, G=2), True),
    (gen.LayerShape(B=3, Cin=6, H=8, W=8, Cout=128, K=1, stride=1, pad=0, G=3), True),
    (gen.LayerShape(B=1, Cin=4, H=31, W=17, Cout=64, K=3, stride=2, pad=0), True),
    # input rows staged in shared memory (a map row a whole number of 16 bytes), CTAs spanning two images
    (gen.LayerShape(B=2, Cin=3, H=40, W=32, Cout=64, K=3, stride=1, pad=1), True),
    (gen.LayerShape(B=1, Cin=3, H=12, W=16, Cout=64, K=3, stride=2, pad=1), True),
    # more than three 128-row tiles per CTA: several rounds (waves), one of them spanning two images
    (gen.LayerShape(B=1, Cin=1, H=250, W=240, Cout=32, K=3, stride=1, pad=1), True),
    (gen.LayerShape(B=2, Cin=3, H=160, W=180, Cout=64, K=3, stride=1, pad=1), True),
    # no mask on the row-per-thread kernel (Cout <= 64)
    (gen.LayerShape(B=2, Cin=2, H=15, W=21, Cout=64, K=3, stride=1, pad=1), False),
    # map rows too wide for the kernel's shared-memory band: every sample read from global memory
    (gen.LayerShape(B=1, Cin=3, H=6, W=1000, Cout=32, K=3, stride=1, pad=1), True),
    # 1x1 and 2x2 kernels on the row-per-thread kernel
    (gen.LayerShape(B=1, Cin=3, H=10, W=17, Cout=32, K=1, stride=1, pad=0), True),
    (gen.LayerShape(B=2, Cin=2, H=11, W=13, Cout=64, K=2, stride=1, pad=0), True),
], ids=lambda v: v if isinstance(v, bool) else "C%dx%dK%ds%dd%dG%d" % (v.Cin, v.Cout, v.K, v.stride, v.dil, v.G))
def test_small_channel_f32_layers(shape, mask, kernel):
    """Float32 layers with few input channels, compared in full: the split-tf32
    tensor-core kernel where it applies, and the CUDA-core kernel (forced with
    DCN_FLAG_NO_TF32) on the same layers."""
    w = gen.Workload("smallc", shape, "f32", seed=9, offset_dist="normal1.5_edges", bias=True)
    d = gen.make_inputs(w)
    if not mask:
        d["mask"] = None
    flags = dcn.DCN_FLAG_NO_TF32 if kernel == "cuda_cores" else 0
    p = dcn._params(d["x"], d["weight"], d["offset"], shape.stride, shape.pad, shape.dil, False, flags)
    expect = "tcgen05_tf32_split" if kernel == "default" and _tf32_split_applies(shape) else "f32_small_channels"
    assert dcn.forward_path(p) == expect
    dd = to_dev(d)
    y = dcn.forward(dd["x"], dd["offset"], dd["mask"], dd["weight"], dd["bias"], shape.stride, shape.pad, shape.dil,
                    flags=flags)
    torch.cuda.synchronize()
    dcn.check_status()
    assert_close(_cpu(y), _oracle_forward(shape, f64(d)), "f32", "y")


@pytest.mark.parametrize("far", [100.0, -3.0e6])
def test_stem_kernel_samples_off_the_band(far):
    """The float32 stem kernel (Cin 3, Cout 64) when every sample misses its
    staged band and the map (offsets of `far`, beyond the clamping bound in one
    case): y equals the bias, which this kernel adds as a contraction column of
    split tf32 parts, so to float32 rounding rather than bit for bit."""
    shape = gen.LayerShape(B=2, Cin=3, H=14, W=20, Cout=64, K=3, stride=1, pad=1)
    w = gen.Workload("smallc", shape, "f32", seed=5, offset_dist="normal1.5_edges", bias=True)
    d = gen.make_inputs(w)
    d["offset"] = torch.full_like(d["offset"], far)
    p = dcn._params(d["x"], d["weight"], d["offset"], shape.stride, shape.pad, shape.dil, False)
    assert dcn.forward_path(p) == "tcgen05_tf32_split"
    dd = to_dev(d)
    y = dcn.forward(dd["x"], dd["offset"], dd["mask"], dd["weight"], dd["bias"], shape.stride, shape.pad, shape.dil)
    torch.cuda.synchronize()
    dcn.check_status()
    expect = np.broadcast_to(d["bias"].double().numpy(), y.shape)
    assert_close(_cpu(y), expect, "f32", "y")
    assert_close(_cpu(y), _oracle_forward(shape, f64(d)), "f32", "y")
