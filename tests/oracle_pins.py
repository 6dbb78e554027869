"""Pins for the float64 oracle: facts that do not come from the oracle itself.

Every ``pin_*`` function takes an oracle library handle (``oracle.load()`` or a
deliberately broken copy built by ``test_oracle_mutants.py``) and raises
AssertionError when the oracle disagrees with the fact it checks:

* a zero offset field with mask = 1 is an ordinary convolution
  (notes "可变形卷积": the plain y(p0) equation is the deformable one with
  dp_n = 0), checked against ``torch.nn.functional.conv2d`` in float64 and a
  brute-force loop nest;
* integer offsets are a convolution whose taps read shifted, zero-filled
  pixels (no interpolation is involved at integer positions);
* a zero mask leaves only the bias (DCNv2 section 3.2: the modulation scalar
  multiplies every sampled value; the tutorial's section 4.2 remark on masks
  near zero);
* bilinear sampling: exact at integer coordinates, the mean of the two or four
  neighbours at half-integers, exact for affine images, and neighbours outside
  the map contribute zero rather than being clamped;
* deformable groups: G groups equal the sum of G single-group layers on the
  channel slices (notes "Deformable Group"), and G copies of one offset field
  equal G = 1;
* the backward is the adjoint of the forward (the forward is linear in x, in
  the weight, in the mask and in the bias), and the offset gradient matches
  finite differences of the forward (notes "计算梯度"), one-sided at exact
  integer coordinates;
* deformable RoI pooling: without offsets it is avg_pool2d of the RoI's k x k
  blocks, whole-pixel shifts move the blocks, half-pixel corners average four
  neighbours, the mask scales each bin, and its backward is the adjoint in x
  and the mask and matches finite differences in the offsets.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle


def _rng(seed):
    return np.random.default_rng(seed)


def _case(seed, B=2, Cin=4, H=7, W=6, Cout=3, K=3, stride=1, pad=1, dil=1, G=1, off_scale=2.0, mask=True, bias=True):
    r = _rng(seed)
    Ho = (H + 2 * pad - dil * (K - 1) - 1) // stride + 1
    Wo = (W + 2 * pad - dil * (K - 1) - 1) // stride + 1
    d = dict(
        x=r.standard_normal((B, H, W, Cin)),
        weight=r.standard_normal((Cout, K, K, Cin)) * 0.5,
        offset=r.uniform(-off_scale, off_scale, (B, 2 * G * K * K, Ho, Wo)),
        mask=r.uniform(0, 1, (B, G * K * K, Ho, Wo)) if mask else None,
        bias=r.standard_normal(Cout) if bias else None,
        grad_y=r.standard_normal((B, Ho, Wo, Cout)),
    )
    return dict(stride=stride, pad=pad, dil=dil, G=G, Ho=Ho, Wo=Wo), d


def _conv2d_ref(x, weight, bias, stride, pad, dil):
    """torch conv2d in float64 on NCHW/OIHW views of the NHWC/OHWI arrays."""
    xt = torch.from_numpy(x).permute(0, 3, 1, 2)
    wt = torch.from_numpy(weight).permute(0, 3, 1, 2)
    bt = None if bias is None else torch.from_numpy(bias)
    y = torch.nn.functional.conv2d(xt, wt, bt, stride=stride, padding=pad, dilation=dil)
    return y.permute(0, 2, 3, 1).numpy()


def _direct_conv_loops(x, weight, bias, stride, pad, dil):
    """Seven nested loops over the plain convolution sum, zero padding."""
    B, H, W, Cin = x.shape
    Cout, K = weight.shape[0], weight.shape[1]
    Ho = (H + 2 * pad - dil * (K - 1) - 1) // stride + 1
    Wo = (W + 2 * pad - dil * (K - 1) - 1) // stride + 1
    y = np.zeros((B, Ho, Wo, Cout))
    for b in range(B):
        for ho in range(Ho):
            for wo in range(Wo):
                for o in range(Cout):
                    acc = 0.0 if bias is None else bias[o]
                    for i in range(K):
                        for j in range(K):
                            r, q = ho * stride - pad + i * dil, wo * stride - pad + j * dil
                            if 0 <= r < H and 0 <= q < W:
                                for c in range(Cin):
                                    acc += weight[o, i, j, c] * x[b, r, q, c]
                    y[b, ho, wo, o] = acc
    return y


# ------------------------------------------------------------------ forward --

def pin_zero_offset_is_conv2d(lib):
    sweep = [
        dict(K=3, stride=1, pad=1, dil=1), dict(K=3, stride=2, pad=1, dil=1), dict(K=1, stride=1, pad=0, dil=1),
        dict(K=5, stride=1, pad=2, dil=1), dict(K=3, stride=1, pad=2, dil=2), dict(K=3, stride=2, pad=0, dil=2),
        dict(K=2, stride=1, pad=0, dil=1),
    ]
    for n, kw in enumerate(sweep):
        for G in (1, 2):
            p, d = _case(100 + n, H=9, W=8, Cin=4, G=G, **kw)
            off = np.zeros_like(d["offset"])
            ones = np.ones_like(d["mask"])
            y = oracle.forward(d["x"], off, ones, d["weight"], d["bias"], p["stride"], p["pad"], p["dil"], G, lib=lib)
            ref = _conv2d_ref(d["x"], d["weight"], d["bias"], p["stride"], p["pad"], p["dil"])
            assert y.shape == ref.shape, (y.shape, ref.shape)
            np.testing.assert_allclose(y, ref, rtol=0, atol=1e-12, err_msg=str(kw))
            y_nomask = oracle.forward(d["x"], off, None, d["weight"], d["bias"], p["stride"], p["pad"], p["dil"], G,
                                      lib=lib)
            np.testing.assert_allclose(y_nomask, ref, rtol=0, atol=1e-12)


def pin_zero_offset_is_direct_loops(lib):
    p, d = _case(7, B=1, Cin=3, H=5, W=6, Cout=2, K=3, stride=2, pad=2, dil=2)
    y = oracle.forward(d["x"], np.zeros_like(d["offset"]), None, d["weight"], d["bias"], 2, 2, 2, 1, lib=lib)
    ref = _direct_conv_loops(d["x"], d["weight"], d["bias"], 2, 2, 2)
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-12)


def _shifted_conv(x, weight, bias, shifts, mvals, stride, pad, dil, G, Ho, Wo):
    """Convolution whose tap k of group g reads x at an extra integer shift
    (dy, dx) = shifts[g][k], zero outside, times the constant mask mvals[g][k]."""
    B, H, W, Cin = x.shape
    Cout, K = weight.shape[0], weight.shape[1]
    Cg = Cin // G
    xp = np.zeros((B, H + 2 * 64, W + 2 * 64, Cin))
    xp[:, 64:64 + H, 64:64 + W, :] = x
    y = np.zeros((B, Ho, Wo, Cout)) + (0.0 if bias is None else bias)
    ho = np.arange(Ho)[:, None]
    wo = np.arange(Wo)[None, :]
    for g in range(G):
        cs = slice(g * Cg, (g + 1) * Cg)
        for i in range(K):
            for j in range(K):
                k = i * K + j
                dy, dx = shifts[g][k]
                rows = ho * stride - pad + i * dil + dy + 64
                cols = wo * stride - pad + j * dil + dx + 64
                patch = xp[:, rows, cols, cs]                  # [B, Ho, Wo, Cg]
                y += mvals[g][k] * np.einsum("bhwc,oc->bhwo", patch, weight[:, i, j, cs])
    return y


def pin_integer_offsets_are_shifted_conv(lib):
    for seed, kw in ((11, dict(K=3, stride=1, pad=1, dil=1, G=1)), (12, dict(K=3, stride=2, pad=1, dil=2, G=2)),
                     (13, dict(K=2, stride=1, pad=0, dil=1, G=2))):
        p, d = _case(seed, Cin=4, H=8, W=7, **kw)
        r = _rng(seed + 1000)
        K, G = kw["K"], kw["G"]
        shifts = [[(int(r.integers(-3, 4)), int(r.integers(-3, 4))) for _ in range(K * K)] for _ in range(G)]
        mvals = [[float(r.uniform(0.1, 1.0)) for _ in range(K * K)] for _ in range(G)]
        off = np.zeros_like(d["offset"])
        mask = np.zeros_like(d["mask"])
        for g in range(G):
            for k in range(K * K):
                off[:, g * 2 * K * K + 2 * k] = shifts[g][k][0]      # channel 2k: row offset
                off[:, g * 2 * K * K + 2 * k + 1] = shifts[g][k][1]  # channel 2k+1: column offset
                mask[:, g * K * K + k] = mvals[g][k]
        y = oracle.forward(d["x"], off, mask, d["weight"], d["bias"], p["stride"], p["pad"], p["dil"], G, lib=lib)
        ref = _shifted_conv(d["x"], d["weight"], d["bias"], shifts, mvals, p["stride"], p["pad"], p["dil"], G,
                            p["Ho"], p["Wo"])
        np.testing.assert_allclose(y, ref, rtol=0, atol=1e-12)


def pin_mask_zero_gives_bias(lib):
    p, d = _case(21, G=2, Cin=4)
    y = oracle.forward(d["x"], d["offset"], np.zeros_like(d["mask"]), d["weight"], d["bias"], 1, 1, 1, 2, lib=lib)
    assert np.array_equal(y, np.broadcast_to(d["bias"], y.shape))


def pin_bilinear_closed_forms(lib):
    r = _rng(31)
    img = r.standard_normal((5, 6, 3))
    for n in range(5):
        for m in range(6):
            assert np.array_equal(oracle.bilinear(img, n, m, lib=lib), img[n, m])
    np.testing.assert_allclose(oracle.bilinear(img, 1.5, 2, lib=lib), (img[1, 2] + img[2, 2]) / 2, atol=1e-15)
    np.testing.assert_allclose(oracle.bilinear(img, 3, 4.5, lib=lib), (img[3, 4] + img[3, 5]) / 2, atol=1e-15)
    np.testing.assert_allclose(oracle.bilinear(img, 2.5, 0.5, lib=lib),
                               (img[2, 0] + img[2, 1] + img[3, 0] + img[3, 1]) / 4, atol=1e-15)
    # bilinear interpolation reproduces an affine image exactly inside the map
    rr, cc = np.meshgrid(np.arange(5), np.arange(6), indexing="ij")
    aff = np.stack([1.5 + 0.25 * rr - 0.75 * cc, -2.0 + 1.0 * rr + 0.5 * cc], axis=-1)
    for py, px in ((0.3, 0.7), (2.9, 4.1), (3.5, 0.01), (1.0, 3.75)):
        np.testing.assert_allclose(oracle.bilinear(aff, py, px, lib=lib),
                                   [1.5 + 0.25 * py - 0.75 * px, -2.0 + py + 0.5 * px], atol=1e-13)


def pin_bilinear_outside_is_zero_not_clamped(lib):
    one = np.ones((4, 5, 1))
    # a quarter of the way above row 0: the row -1 neighbours are outside and count zero
    np.testing.assert_allclose(oracle.bilinear(one, -0.25, 2.0, lib=lib), [0.75], atol=1e-15)
    np.testing.assert_allclose(oracle.bilinear(one, 1.0, 4.5, lib=lib), [0.5], atol=1e-15)
    np.testing.assert_allclose(oracle.bilinear(one, -0.5, -0.5, lib=lib), [0.25], atol=1e-15)
    for py, px in ((-1.0, 2.0), (4.0, 1.0), (1.0, -1.0), (2.0, 5.0), (-3.2, 1.1), (9.0, 9.0)):
        assert oracle.bilinear(one, py, px, lib=lib)[0] == 0.0
    # the sample just inside the last row keeps its inside share only
    np.testing.assert_allclose(oracle.bilinear(one, 3.25, 0.0, lib=lib), [0.75], atol=1e-15)


def pin_groups_decompose(lib):
    p, d = _case(41, Cin=6, G=3, K=3, Cout=4)
    y = oracle.forward(d["x"], d["offset"], d["mask"], d["weight"], d["bias"], 1, 1, 1, 3, lib=lib)
    K2 = 9
    acc = np.zeros_like(y) + d["bias"]
    for g in range(3):
        cs = slice(2 * g, 2 * g + 2)
        acc += oracle.forward(d["x"][..., cs], d["offset"][:, g * 2 * K2:(g + 1) * 2 * K2],
                              d["mask"][:, g * K2:(g + 1) * K2], d["weight"][..., cs], None, 1, 1, 1, 1, lib=lib)
    np.testing.assert_allclose(y, acc, rtol=0, atol=1e-12)


def pin_group_copies_equal_one_group(lib):
    p, d = _case(42, Cin=4, G=1)
    y1 = oracle.forward(d["x"], d["offset"], d["mask"], d["weight"], d["bias"], 1, 1, 1, 1, lib=lib)
    y2 = oracle.forward(d["x"], np.concatenate([d["offset"]] * 2, 1), np.concatenate([d["mask"]] * 2, 1),
                        d["weight"], d["bias"], 1, 1, 1, 2, lib=lib)
    np.testing.assert_allclose(y1, y2, rtol=0, atol=1e-12)


def pin_linear_in_x_weight_mask(lib):
    p, d = _case(43, G=2, Cin=4, stride=2, dil=2, pad=2)
    f = lambda x, w, m: oracle.forward(x, d["offset"], m, w, None, 2, 2, 2, 2, lib=lib)
    r = _rng(44)
    x2 = r.standard_normal(d["x"].shape)
    np.testing.assert_allclose(f(d["x"] + 2 * x2, d["weight"], d["mask"]),
                               f(d["x"], d["weight"], d["mask"]) + 2 * f(x2, d["weight"], d["mask"]), atol=1e-12)
    w2 = r.standard_normal(d["weight"].shape)
    np.testing.assert_allclose(f(d["x"], d["weight"] - w2, d["mask"]),
                               f(d["x"], d["weight"], d["mask"]) - f(d["x"], w2, d["mask"]), atol=1e-12)
    np.testing.assert_allclose(f(d["x"], d["weight"], 3 * d["mask"]), 3 * f(d["x"], d["weight"], d["mask"]),
                               atol=1e-12)


# ----------------------------------------------------------------- backward --

def pin_backward_adjoint_identities(lib):
    for seed, kw in ((51, dict(G=1)), (52, dict(G=2, stride=2, dil=2, pad=2, K=3)), (53, dict(G=1, K=2, pad=0))):
        p, d = _case(seed, Cin=4, Cout=3, **kw)
        a = (p["stride"], p["pad"], p["dil"], p["G"])
        y = oracle.forward(d["x"], d["offset"], d["mask"], d["weight"], d["bias"], *a, lib=lib)
        g = oracle.backward(d["x"], d["offset"], d["mask"], d["weight"], d["grad_y"], *a, lib=lib)
        lhs = float(np.sum(d["grad_y"] * (y - d["bias"])))
        tol = 1e-10 * (1 + abs(lhs))
        assert abs(lhs - float(np.sum(g["grad_x"] * d["x"]))) < tol
        assert abs(lhs - float(np.sum(g["grad_weight"] * d["weight"]))) < tol
        assert abs(lhs - float(np.sum(g["grad_mask"] * d["mask"]))) < tol
        np.testing.assert_allclose(g["grad_bias"], d["grad_y"].sum(axis=(0, 1, 2)), atol=1e-12)
        # the same identity tap by tap for the mask (y - b is linear in each m_k separately)
        gm_full = g["grad_mask"]
        for k in (0, d["mask"].shape[1] - 1):
            m2 = d["mask"].copy()
            m2[:, k] = 0.0
            y2 = oracle.forward(d["x"], d["offset"], m2, d["weight"], d["bias"], *a, lib=lib)
            np.testing.assert_allclose(float(np.sum(d["grad_y"] * (y - y2))),
                                       float(np.sum(gm_full[:, k] * d["mask"][:, k])), atol=tol)


def _loss(lib, d, a, **over):
    e = dict(d)
    e.update(over)
    y = oracle.forward(e["x"], e["offset"], e["mask"], e["weight"], e["bias"], *a, lib=lib)
    return float(np.sum(d["grad_y"] * y))


def pin_backward_finite_differences(lib):
    p, d = _case(61, B=1, Cin=3, Cout=2, H=6, W=5, G=1, off_scale=2.5)
    a = (p["stride"], p["pad"], p["dil"], p["G"])
    # keep every sample away from integer coordinates so central differences are clean
    d["offset"] = np.round(d["offset"] * 8) / 8 + 1.0 / 16
    g = oracle.backward(d["x"], d["offset"], d["mask"], d["weight"], d["grad_y"], *a, lib=lib)
    r = _rng(62)
    for name in ("x", "weight", "mask", "bias", "offset"):
        arr = d[name]
        h = 1e-6 if name == "offset" else 0.5       # the loss is linear in all but the offsets
        gname = {"x": "grad_x", "weight": "grad_weight", "mask": "grad_mask", "bias": "grad_bias",
                 "offset": "grad_offset"}[name]
        for _ in range(12):
            idx = tuple(int(r.integers(0, n)) for n in arr.shape)
            up, dn = arr.copy(), arr.copy()
            up[idx] += h
            dn[idx] -= h
            fd = (_loss(lib, d, a, **{name: up}) - _loss(lib, d, a, **{name: dn})) / (2 * h)
            np.testing.assert_allclose(g[gname][idx], fd, rtol=1e-6, atol=1e-7, err_msg="%s %s" % (name, idx))


def pin_offset_gradient_one_sided_at_integers(lib):
    p, d = _case(63, B=1, Cin=2, Cout=2, H=6, W=6, G=1)
    a = (p["stride"], p["pad"], p["dil"], p["G"])
    d["offset"] = np.round(d["offset"])            # every sample exactly on the grid
    d["offset"][0, 0, 0, 0] = 0.0                # tap (0,0) of pixel (0,0) has base row -1: py = -1 exactly
    g = oracle.backward(d["x"], d["offset"], d["mask"], d["weight"], d["grad_y"], *a, lib=lib)
    r = _rng(64)
    picks = [(0, 0, 0, 0)] + [tuple(int(r.integers(0, n)) for n in d["offset"].shape) for _ in range(15)]
    for idx in picks:
        h = 1e-6
        up = d["offset"].copy()
        up[idx] += h
        fd = (_loss(lib, d, a, offset=up) - _loss(lib, d, a)) / h   # right-hand difference
        np.testing.assert_allclose(g["grad_offset"][idx], fd, rtol=1e-5, atol=1e-6, err_msg=str(idx))


def pin_sampled_entries_match_full(lib):
    """The sampled-entry routines equal the corresponding entries of the full
    backward/forward (both already pinned above)."""
    p, d = _case(71, B=2, Cin=4, Cout=3, G=2, stride=2, pad=1)
    a = (p["stride"], p["pad"], p["dil"], p["G"])
    y = oracle.forward(d["x"], d["offset"], d["mask"], d["weight"], d["bias"], *a, lib=lib)
    g = oracle.backward(d["x"], d["offset"], d["mask"], d["weight"], d["grad_y"], *a, lib=lib)
    r = _rng(72)
    P = y.shape[0] * y.shape[1] * y.shape[2]
    pix = r.choice(P, 7, replace=False)
    np.testing.assert_allclose(oracle.forward(d["x"], d["offset"], d["mask"], d["weight"], d["bias"], *a,
                                              pixels=pix, lib=lib), y.reshape(P, -1)[pix], atol=1e-13)
    goff, gm = oracle.grad_offset_mask_at(d["x"], d["offset"], d["mask"], d["weight"], d["grad_y"], pix, *a, lib=lib)
    B, C2, Ho, Wo = g["grad_offset"].shape
    np.testing.assert_allclose(goff, g["grad_offset"].transpose(0, 2, 3, 1).reshape(P, C2)[pix], atol=1e-12)
    np.testing.assert_allclose(gm, g["grad_mask"].transpose(0, 2, 3, 1).reshape(P, -1)[pix], atol=1e-12)
    we = r.choice(g["grad_weight"].size, 9, replace=False)
    np.testing.assert_allclose(oracle.grad_weight_at(d["x"], d["offset"], d["mask"], d["grad_y"], d["weight"].shape,
                                                     we, *a, lib=lib), g["grad_weight"].reshape(-1)[we], atol=1e-12)
    xe = r.choice(g["grad_x"].size, 9, replace=False)
    np.testing.assert_allclose(oracle.grad_x_at(d["x"].shape, d["offset"], d["mask"], d["weight"], d["grad_y"], xe,
                                                *a, lib=lib), g["grad_x"].reshape(-1)[xe], atol=1e-12)


# ------------------------------------------------ offset/mask predictor --

def pin_predictor_is_conv2d_split_sigmoid(lib):
    """The predictor is torch's own conv2d (float64) with the layer's geometry;
    its first 2GK^2 output channels are the offsets and the rest, through
    torch.sigmoid, the masks. Swept over K, stride, padding, dilation, groups."""
    for n, (K, stride, pad, dil, G) in enumerate([(3, 1, 1, 1, 1), (3, 2, 1, 1, 2), (1, 1, 0, 1, 1),
                                                   (3, 1, 2, 2, 1), (5, 1, 2, 1, 1)]):
        r = _rng(200 + n)
        B, H, W, Cin, NC = 2, 7, 9, 3, 3 * G * K * K
        x = r.standard_normal((B, H, W, Cin))
        w = r.standard_normal((NC, K, K, Cin)) * 0.3
        b = r.standard_normal(NC)
        off, mask = oracle.predict_offset_mask(x, w, b, K, stride, pad, dil, G, lib=lib)
        ref = _conv2d_ref(x, w, b, stride, pad, dil).transpose(0, 3, 1, 2)  # [B, NC, Ho, Wo]
        NO = 2 * G * K * K
        assert off.shape == ref[:, :NO].shape and mask.shape == ref[:, NO:].shape
        assert np.allclose(off, ref[:, :NO], rtol=1e-12, atol=1e-12)
        assert np.allclose(mask, torch.sigmoid(torch.from_numpy(ref[:, NO:])).numpy(), rtol=1e-12, atol=1e-12)


def pin_predictor_bias_only(lib):
    """Zero weights: the offsets equal the bias everywhere; with no bias the
    masks are exactly 1/2 (the logistic function at 0)."""
    r = _rng(210)
    K, G = 3, 2
    NC = 3 * G * K * K
    x = r.standard_normal((1, 6, 5, 4))
    w = np.zeros((NC, K, K, 4))
    b = r.standard_normal(NC)
    off, mask = oracle.predict_offset_mask(x, w, b, K, 1, 1, 1, G, lib=lib)
    assert np.array_equal(off, np.broadcast_to(b[:2 * G * K * K, None, None], off.shape[1:])[None].repeat(1, 0))
    off0, mask0 = oracle.predict_offset_mask(x, w, None, K, 1, 1, 1, G, lib=lib)
    assert np.all(off0 == 0.0) and np.all(mask0 == 0.5)


# --------------------------------------------------- deformable RoI pooling --

def _avg_pool_blocks(x, b, y1, x1, h, w, k, pad=0):
    """torch avg_pool2d (float64) of the h x w block at (y1, x1) of image b, cut
    into k x k equal blocks; the image is zero-padded by `pad` first, so blocks
    reaching outside the map average zeros there. Returns [k, k, C]."""
    img = torch.from_numpy(x[b]).permute(2, 0, 1)[None]  # [1, C, H, W]
    img = torch.nn.functional.pad(img, (pad, pad, pad, pad))
    crop = img[:, :, y1 + pad:y1 + pad + h, x1 + pad:x1 + pad + w]
    out = torch.nn.functional.avg_pool2d(crop, kernel_size=(h // k, w // k))
    return out[0].permute(1, 2, 0).numpy()


def pin_droi_plain_is_avg_pool(lib):
    """Without offsets, a RoI with integer corners whose sides are multiples of k
    pools to torch's avg_pool2d of its k x k blocks, zeros outside the map
    (notes, "可变形ROI pooling": each output averages its bin's pixels)."""
    r = _rng(300)
    x = r.standard_normal((2, 9, 11, 3))
    k = 3
    rois = np.array([[0, 2, 0, 8, 9], [1, 0, 3, 9, 9], [1, -2, -1, 7, 5], [0, 6, 4, 12, 10]], dtype=float)
    y = oracle.droi_pool_forward(x, rois, None, None, k, lib=lib)
    for n, (b, x1, y1, x2, y2) in enumerate(rois.astype(int)):
        ref = _avg_pool_blocks(x, b, y1, x1, y2 - y1, x2 - x1, k, pad=4)
        assert np.allclose(y[n], ref, rtol=1e-12, atol=1e-12), n


def pin_droi_integer_shifts_move_blocks(lib):
    """Offsets whose shift gamma*off*h (and *w) is a whole number of pixels move
    each bin's block by that many pixels: the mean of the moved block, zeros
    outside the map; normalised offsets scale with the RoI's size and gamma."""
    r = _rng(301)
    x = r.standard_normal((1, 10, 12, 2))
    k, gamma = 2, 0.5
    rois = np.array([[0, 2, 1, 10, 9]], dtype=float)  # w = 8, h = 8: blocks of 4 x 4
    h = w = 8
    sh = r.integers(-3, 4, size=(k * k, 2))
    off = np.zeros((1, 2 * k * k))
    off[0, 0::2] = sh[:, 0] / (gamma * h)
    off[0, 1::2] = sh[:, 1] / (gamma * w)
    y = oracle.droi_pool_forward(x, rois, off, None, k, gamma, lib=lib)
    xp = np.pad(x[0], ((6, 6), (6, 6), (0, 0)))
    for i in range(k):
        for j in range(k):
            t = i * k + j
            r0, c0 = 1 + i * 4 + sh[t, 0] + 6, 2 + j * 4 + sh[t, 1] + 6
            ref = xp[r0:r0 + 4, c0:c0 + 4].mean(axis=(0, 1))
            assert np.allclose(y[0, i, j], ref, rtol=1e-12, atol=1e-12), (i, j)


def pin_droi_half_pixel_corners_average_neighbours(lib):
    """A RoI whose corners sit on half-integers samples midway between four
    pixels: the pooled values equal avg_pool2d of the 2 x 2 box-filtered map."""
    r = _rng(302)
    x = r.standard_normal((1, 8, 8, 2))
    k = 2
    rois = np.array([[0, 1.5, 0.5, 5.5, 6.5]], dtype=float)  # w = 4, h = 6
    y = oracle.droi_pool_forward(x, rois, None, None, k, lib=lib)
    img = torch.from_numpy(x[0]).permute(2, 0, 1)[:, None]  # [C, 1, H, W]
    box = torch.nn.functional.conv2d(img, torch.full((1, 1, 2, 2), 0.25, dtype=torch.float64))  # [C,1,H-1,W-1]
    # sample (0.5 + u, 1.5 + v) is the box filter at (u, v + 1)
    crop = box[:, :, 0:6, 1:5]
    ref = torch.nn.functional.avg_pool2d(crop, kernel_size=(3, 2))[:, 0].permute(1, 2, 0).numpy()
    assert np.allclose(y[0], ref, rtol=1e-12, atol=1e-12)


def pin_droi_mask_scales_and_gamma_zero_is_plain(lib):
    """The per-bin mask multiplies the bin's output (DCNv2 section 3.2); gamma = 0
    removes every offset."""
    r = _rng(303)
    x = r.standard_normal((2, 7, 9, 3))
    k = 3
    rois = np.array([[0, 0.3, 1.2, 7.9, 6.1], [1, 2, 2, 5, 5]], dtype=float)
    off = r.uniform(-0.4, 0.4, (2, 2 * k * k))
    mask = r.uniform(0, 1, (2, k * k))
    y1 = oracle.droi_pool_forward(x, rois, off, None, k, 0.3, lib=lib)
    ym = oracle.droi_pool_forward(x, rois, off, mask, k, 0.3, lib=lib)
    assert np.allclose(ym, y1 * mask.reshape(2, k, k, 1), rtol=1e-12, atol=1e-12)
    assert np.array_equal(oracle.droi_pool_forward(x, rois, off, None, k, 0.0, lib=lib),
                          oracle.droi_pool_forward(x, rois, None, None, k, lib=lib))


def pin_droi_backward_adjoint_and_finite_differences(lib):
    """The backward is the adjoint of the forward in x and in the mask (the
    forward is linear in both), and its offset gradient matches central finite
    differences of the forward."""
    r = _rng(304)
    x = r.standard_normal((2, 8, 9, 3))
    k, gamma = 3, 0.2
    rois = np.array([[0, 0.7, 1.3, 7.6, 6.9], [1, 1.2, 0.4, 8.8, 7.7], [1, 3.1, 2.2, 5.3, 4.9]], dtype=float)
    off = r.uniform(-0.5, 0.5, (3, 2 * k * k))
    mask = r.uniform(0, 1, (3, k * k))
    gy = r.standard_normal((3, k, k, 3))
    y = oracle.droi_pool_forward(x, rois, off, mask, k, gamma, lib=lib)
    gx, goff, gm = oracle.droi_pool_backward(x, rois, off, mask, gy, k, gamma, lib=lib)
    lhs = float((gy * y).sum())
    assert abs(lhs - float((gx * x).sum())) <= 1e-10 * (1 + abs(lhs))
    assert abs(lhs - float((gm * mask).sum())) <= 1e-10 * (1 + abs(lhs))
    eps = 1e-6
    for n in range(3):
        for q in r.choice(2 * k * k, 6, replace=False):
            op, om = off.copy(), off.copy()
            op[n, q] += eps
            om[n, q] -= eps
            fd = ((gy * oracle.droi_pool_forward(x, rois, op, mask, k, gamma, lib=lib)).sum() -
                  (gy * oracle.droi_pool_forward(x, rois, om, mask, k, gamma, lib=lib)).sum()) / (2 * eps)
            assert abs(fd - goff[n, q]) <= 1e-6 * (1 + abs(fd)), (n, q, fd, goff[n, q])


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
