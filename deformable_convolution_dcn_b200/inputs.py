"""Seeded synthetic inputs for the DCNv2 layer shapes used by tests and the bench.

This module only draws random numbers and lays them out; it holds none of the
convolution's arithmetic, so both the CUDA library and the float64 oracle can
be fed from it. Every tensor is drawn on the CPU with ``torch.Generator`` in
logical order (x as [B, Cin, H, W], weight as [Cout, Cin, K, K]) and then
permuted to the library layouts:

    x       [B, H, W, Cin]          offset [B, 2*G*K*K, Ho, Wo]
    weight  [Cout, K, K, Cin]       mask   [B, G*K*K, Ho, Wo]
    bias    [Cout]                  grad_y [B, Ho, Wo, Cout]

The shapes are the ResNet-50 bottleneck 3x3 convolutions that DCNv2 replaces in
stages conv3..conv5 (the mmdetection ``stage_with_dcn`` walkthrough; DCNv2
section 3.1) and the 224x224 RGB example layer of the torchvision tutorial
(section 2.2). The value distributions follow the tutorial: Kaiming-normal
weights (section 2.1 table), offsets limited by 0.5*tanh (section 2.2 and the
module's forward), masks through a sigmoid (DCNv2 section 3.2).
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class LayerShape:
    B: int
    Cin: int
    H: int
    W: int
    Cout: int
    K: int = 3
    stride: int = 1
    pad: int = 1
    dil: int = 1
    G: int = 1

    @property
    def Ho(self) -> int:
        return (self.H + 2 * self.pad - self.dil * (self.K - 1) - 1) // self.stride + 1

    @property
    def Wo(self) -> int:
        return (self.W + 2 * self.pad - self.dil * (self.K - 1) - 1) // self.stride + 1

    @property
    def P(self) -> int:
        """Output pixels B*Ho*Wo (the GEMM M)."""
        return self.B * self.Ho * self.Wo

    def flops(self) -> float:
        """2*M*N*K of the dense contraction, M = B*Ho*Wo, N = Cout, K = Cin*K*K."""
        return 2.0 * self.P * self.Cout * self.Cin * self.K * self.K


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    shape: LayerShape
    dtype: str                    # "f32" or "bf16": the dtype of every input and of y
    seed: int
    x_dist: str = "normal"
    w_dist: str = "kaiming"       # "kaiming" (std sqrt(2/fan_in)) or "normal0.1"
    offset_dist: str = "normal1.5"  # "uniform2.5" | "tanh0.5" | "normal1.5" | "normal1.5_edges"
    mask_dist: str = "sigmoid"    # "uniform" | "sigmoid" | "none"
    bias: bool = False
    backward: bool = False
    description: str = ""


WORKLOADS = {
    "tiny": Workload(
        "tiny", LayerShape(B=1, Cin=4, H=16, W=16, Cout=8), "f32", seed=0,
        w_dist="normal0.1", offset_dist="uniform2.5", mask_dist="uniform", bias=True, backward=True,
        description="tiny DCNv2 forward+backward fp32, B1 Cin4 16x16 Cout8 K3 s1 p1 G1, bias"),
    "stem": Workload(
        "stem", LayerShape(B=1, Cin=3, H=224, W=224, Cout=64), "f32", seed=1,
        offset_dist="tanh0.5", mask_dist="sigmoid",
        description="224x224 RGB stem-like DCNv2 forward fp32, B1 Cin3 Cout64 K3 s1 p1 G1"),
    "conv4": Workload(
        "conv4", LayerShape(B=8, Cin=256, H=50, W=50, Cout=256), "bf16", seed=2,
        description="ResNet-50 conv4 3x3 DCNv2 forward bf16, B8 Cin=Cout=256 50x50 K3 s1 p1 G1"),
    "conv3_s2": Workload(
        "conv3_s2", LayerShape(B=8, Cin=128, H=200, W=200, Cout=128, stride=2), "bf16", seed=3,
        description="ResNet-50 conv3 down-sample DCNv2 forward bf16, B8 Cin=Cout=128 200x200->100x100 s2 p1"),
    "conv5_d2g4": Workload(
        "conv5_d2g4", LayerShape(B=8, Cin=512, H=25, W=25, Cout=512, pad=2, dil=2, G=4), "bf16", seed=4,
        description="ResNet-50 conv5 DCNv2 forward bf16, B8 Cin=Cout=512 25x25 s1 p2 d2 G4"),
    "conv4_v1": Workload(
        "conv4_v1", LayerShape(B=8, Cin=256, H=50, W=50, Cout=256), "bf16", seed=6, mask_dist="none",
        description="ResNet-50 conv4 3x3 DCNv1 forward bf16 (no modulation mask), B8 Cin=Cout=256 50x50 K3 s1 p1 G1"),
    "conv4_k5": Workload(
        "conv4_k5", LayerShape(B=8, Cin=256, H=50, W=50, Cout=256, K=5, pad=2), "bf16", seed=7,
        description="conv4-sized 5x5 DCNv2 forward bf16 (50 offset channels), B8 Cin=Cout=256 50x50 K5 s1 p2 G1"),
    "conv4_k7": Workload(
        "conv4_k7", LayerShape(B=8, Cin=256, H=50, W=50, Cout=256, K=7, pad=3), "bf16", seed=8,
        description="conv4-sized 7x7 DCNv2 forward bf16 (98 offset channels), B8 Cin=Cout=256 50x50 K7 s1 p3 G1"),
    "conv4_bwd": Workload(
        "conv4_bwd", LayerShape(B=8, Cin=256, H=50, W=50, Cout=256), "bf16", seed=5,
        offset_dist="normal1.5_edges", backward=True,
        description="full backward of the conv4 shape, bf16 activations, fp32 gradients; offsets include "
                    "samples exactly on integer coordinates and outside the map"),
}


def torch_dtype(dtype: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[dtype]


def _draw_offsets(g: torch.Generator, s: LayerShape, dist: str) -> torch.Tensor:
    n = (s.B, 2 * s.G * s.K * s.K, s.Ho, s.Wo)
    if dist == "uniform2.5":
        return (torch.rand(n, generator=g) * 5.0) - 2.5
    if dist == "tanh0.5":
        return 0.5 * torch.tanh(torch.randn(n, generator=g))
    if dist in ("normal1.5", "normal1.5_edges"):
        off = 1.5 * torch.randn(n, generator=g)
        if dist == "normal1.5_edges":
            u = torch.rand(n, generator=g)
            # 10 % land exactly on integer coordinates (the base position is an integer)
            off = torch.where(u < 0.10, torch.round(off), off)
            # 2 % jump outside the map entirely
            sign = torch.where(torch.rand(n, generator=g) < 0.5, -1.0, 1.0)
            off = torch.where((u >= 0.10) & (u < 0.12), sign * float(max(s.H, s.W) + 2), off)
            # a few rows sample exactly at row -1 / column -1 (one-sided border derivative)
            for t in range(min(32, s.B * s.Ho * s.Wo)):
                b = t % s.B
                ho = (7 * t) % s.Ho
                wo = (13 * t) % s.Wo
                k = t % (s.K * s.K)
                gg = t % s.G
                i, j = divmod(k, s.K)
                base_y = ho * s.stride - s.pad + i * s.dil
                base_x = wo * s.stride - s.pad + j * s.dil
                ch = gg * 2 * s.K * s.K + 2 * k
                if t % 2 == 0:
                    off[b, ch, ho, wo] = -float(base_y + 1)
                else:
                    off[b, ch + 1, ho, wo] = -float(base_x + 1)
        return off
    raise ValueError(dist)


def make_inputs(w: Workload | str, device="cpu", seed: int | None = None, shape: LayerShape | None = None):
    """Inputs of a workload (or of ``shape`` with the workload's distributions).

    Returns a dict of tensors in the library layouts and in the workload dtype:
    x, offset, mask (None when the workload has no mask), weight, bias (None
    without bias) and, for backward workloads, grad_y.
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    s = shape or w.shape
    g = torch.Generator().manual_seed(w.seed if seed is None else seed)
    dt = torch_dtype(w.dtype)
    x = torch.randn((s.B, s.Cin, s.H, s.W), generator=g).permute(0, 2, 3, 1).contiguous()
    fan_in = s.Cin * s.K * s.K
    if w.w_dist == "kaiming":
        wt = torch.randn((s.Cout, s.Cin, s.K, s.K), generator=g) * math.sqrt(2.0 / fan_in)
    elif w.w_dist == "normal0.1":
        wt = torch.randn((s.Cout, s.Cin, s.K, s.K), generator=g) * 0.1
    else:
        raise ValueError(w.w_dist)
    wt = wt.permute(0, 2, 3, 1).contiguous()
    off = _draw_offsets(g, s, w.offset_dist)
    mshape = (s.B, s.G * s.K * s.K, s.Ho, s.Wo)
    if w.mask_dist == "uniform":
        mask = torch.rand(mshape, generator=g)
    elif w.mask_dist == "sigmoid":
        mask = torch.sigmoid(torch.randn(mshape, generator=g))
    elif w.mask_dist == "none":
        mask = None
    else:
        raise ValueError(w.mask_dist)
    bias = torch.randn((s.Cout,), generator=g) if w.bias else None
    out = {"x": x, "offset": off, "mask": mask, "weight": wt, "bias": bias}
    if w.backward:
        out["grad_y"] = torch.randn((s.B, s.Cout, s.Ho, s.Wo), generator=g).permute(0, 2, 3, 1).contiguous()
    return {k: (None if v is None else v.to(dt).to(device)) for k, v in out.items()}


def random_case(seed: int, dtype: str = "f32", B=None, Cin=None, H=None, W=None, Cout=None, K=None, stride=None,
                pad=None, dil=None, G=None, offset_scale=2.0, with_mask=True, with_bias=True, backward=True,
                device="cpu"):
    """A small random layer (for sweeps over K, stride, pad, dil, G and ragged sizes).

    Unspecified sizes are drawn from the generator; offsets ~ U(-offset_scale, offset_scale)
    so that samples fall off-grid and outside the map.
    """
    g = torch.Generator().manual_seed(seed)
    pick = lambda v, choices: v if v is not None else choices[int(torch.randint(len(choices), (1,), generator=g))]
    G = pick(G, [1, 1, 2])
    K = pick(K, [1, 3, 3, 5])
    dil = pick(dil, [1, 1, 2])
    stride = pick(stride, [1, 1, 2])
    pad = pick(pad, [0, (K // 2) * dil, K // 2])
    Cin = pick(Cin, [c * G for c in (1, 3, 4, 8)])
    Cout = pick(Cout, [1, 5, 8, 16])
    B = pick(B, [1, 2])
    H = pick(H, [5, 7, 9, 12])
    W = pick(W, [4, 6, 9, 11])
    s = LayerShape(B=B, Cin=Cin, H=H, W=W, Cout=Cout, K=K, stride=stride, pad=pad, dil=dil, G=G)
    if s.Ho <= 0 or s.Wo <= 0:
        s = dataclasses.replace(s, pad=(K - 1) * dil)
    dt = torch_dtype(dtype)
    x = torch.randn((s.B, s.Cin, s.H, s.W), generator=g).permute(0, 2, 3, 1).contiguous()
    wt = (torch.randn((s.Cout, s.Cin, s.K, s.K), generator=g) * 0.3).permute(0, 2, 3, 1).contiguous()
    off = (torch.rand((s.B, 2 * s.G * s.K * s.K, s.Ho, s.Wo), generator=g) * 2.0 - 1.0) * offset_scale
    mask = torch.rand((s.B, s.G * s.K * s.K, s.Ho, s.Wo), generator=g) if with_mask else None
    bias = torch.randn((s.Cout,), generator=g) if with_bias else None
    out = {"x": x, "offset": off, "mask": mask, "weight": wt, "bias": bias}
    if backward:
        out["grad_y"] = torch.randn((s.B, s.Ho, s.Wo, s.Cout), generator=g)
    return s, {k: (None if v is None else v.to(dt).to(device)) for k, v in out.items()}


def predictor_inputs(seed: int, s: LayerShape, dtype: str = "f32", bias: bool = True, device="cpu"):
    """Inputs of a layer's offset/mask predictor: x [B, H, W, Cin], w_pred
    [3*G*K*K, K, K, Cin] and b_pred [3*G*K*K] (None without bias).

    DCNv2 starts the predictor at zero weights (DCNv2 section 3.2); a trained
    one does not stay there, so the weights here are normal with std
    1/sqrt(Cin*K*K) (outputs of unit scale: offsets of about one pixel, masks
    spread over (0, 1)) and the bias is normal with std 0.5. s.Cout is unused.
    """
    g = torch.Generator().manual_seed(seed)
    nc = 3 * s.G * s.K * s.K
    x = torch.randn((s.B, s.Cin, s.H, s.W), generator=g).permute(0, 2, 3, 1).contiguous()
    w = torch.randn((nc, s.Cin, s.K, s.K), generator=g) / math.sqrt(s.Cin * s.K * s.K)
    b = torch.randn((nc,), generator=g) * 0.5 if bias else None
    out = {"x": x, "w_pred": w.permute(0, 2, 3, 1).contiguous(), "b_pred": b}
    dt = torch_dtype(dtype)
    return {k: (None if v is None else v.to(dt).to(device)) for k, v in out.items()}


def roi_inputs(seed: int, B: int, H: int, W: int, C: int, R: int, k: int, dtype: str = "f32", offsets: bool = True,
               mask: bool = True, max_side: float | None = None, device="cpu"):
    """Inputs of deformable RoI pooling: x [B, H, W, C] ~ N(0, 1); R RoIs (b, x1,
    y1, x2, y2) float32 with corners on a 1/8-pixel grid, sides up to max_side
    (default the map's), some reaching past the map's edges; normalised offsets
    [R, 2k^2] ~ U(-0.3, 0.3) rounded to 1/64; masks [R, k^2] ~ U(0, 1)."""
    g = torch.Generator().manual_seed(seed)
    dt = torch_dtype(dtype)
    x = torch.randn((B, C, H, W), generator=g).permute(0, 2, 3, 1).contiguous()
    side = max_side or float(max(H, W))
    b = torch.randint(0, B, (R,), generator=g).float()
    cx = torch.rand(R, generator=g) * (W + 2) - 1
    cy = torch.rand(R, generator=g) * (H + 2) - 1
    ww = torch.rand(R, generator=g) * side
    hh = torch.rand(R, generator=g) * side
    q = lambda v: torch.round(v * 8) / 8
    rois = torch.stack([b, q(cx - ww / 2), q(cy - hh / 2), q(cx + ww / 2), q(cy + hh / 2)], dim=1)
    # offsets on a 1/64 grid: with dyadic gamma every sample position is exact in float32 and float64
    off = (torch.round((torch.rand((R, 2 * k * k), generator=g) * 0.6 - 0.3) * 64) / 64) if offsets else None
    m = torch.rand((R, k * k), generator=g) if mask else None
    gy = torch.randn((R, k, k, C), generator=g)
    out = {"x": x.to(dt), "rois": rois, "offset": None if off is None else off.to(dt),
           "mask": None if m is None else m.to(dt), "grad_y": gy.to(dt)}
    return {n: (None if v is None else v.to(device)) for n, v in out.items()}


def as_f64(t):
    """numpy float64 copy of a tensor's stored values (None passes through)."""
    if t is None:
        return None
    return t.detach().to("cpu", torch.float64).numpy()
