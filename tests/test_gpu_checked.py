"""The range-checked build (DCN_CHECKED, libdcn_b200_checked.so) on the GPU:
every checked gather and scatter of the tensor-core forward, backward_data and
backward_weight kernels, and the float32 stem kernel's band and neighbour
reads, stays inside its buffer on layers whose samples reach
the map's edges and beyond (the status word stays clear), and the forward's
output equals the regular build's bit for bit (the checks change no value).
The checked build runs in a child process (a process loads one build)."""
import json
import os
import subprocess
import sys

import pytest
import torch

import deformable_convolution_dcn_b200 as dcn
from deformable_convolution_dcn_b200 import inputs as gen

from parity import assert_close

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SHAPES = {
    "tmem": gen.LayerShape(B=2, Cin=64, H=12, W=11, Cout=64),               # fwd_tc_ts.cu
    "smem": gen.LayerShape(B=1, Cin=32, H=10, W=9, Cout=272),               # fwd_tc.cu (Cout > 256)
    "dil2g2": gen.LayerShape(B=1, Cin=64, H=9, W=13, Cout=96, pad=2, dil=2, G=2),
    "stem_f32": gen.LayerShape(B=2, Cin=3, H=40, W=32, Cout=64),            # fwd_f32_stem.cu (band in shared memory)
}
DTYPE = {"stem_f32": "f32"}

CHILD = r"""
import json, sys, torch
sys.path.insert(0, sys.argv[1])
import deformable_convolution_dcn_b200 as dcn
from deformable_convolution_dcn_b200 import inputs as gen
shapes, dtypes = json.loads(sys.argv[2]); out = {}
for name, kw in shapes.items():
    s = gen.LayerShape(**kw)
    w = gen.Workload("chk", s, dtypes.get(name, "bf16"), seed=5, offset_dist="normal1.5_edges", bias=True)
    d = {k: (None if v is None else v.cuda()) for k, v in gen.make_inputs(w).items()}
    a = (s.stride, s.pad, s.dil)
    y = dcn.forward(d["x"], d["offset"], d["mask"], d["weight"], d["bias"], *a)
    gy = torch.randn(y.shape, generator=torch.Generator().manual_seed(3)).to(y.dtype).cuda()
    gx, goff, gm = dcn.backward_data(d["x"], d["offset"], d["mask"], d["weight"], gy, *a)
    gw, gb = dcn.backward_weight(d["x"], d["offset"], d["mask"], gy, tuple(d["weight"].shape), *a)
    torch.cuda.synchronize()
    dcn.check_status()
    out[name] = {k: v.cpu() for k, v in dict(y=y, gx=gx, goff=goff, gm=gm, gw=gw, gb=gb).items()}
torch.save(out, sys.argv[3])
print("ok")
"""


def test_checked_build_runs_clean_and_matches(tmp_path):
    from deformable_convolution_dcn_b200 import build
    build.build_checked()
    shapes = {k: {f: getattr(v, f) for f in ("B", "Cin", "H", "W", "Cout", "K", "stride", "pad", "dil", "G")}
              for k, v in SHAPES.items()}
    dst = str(tmp_path / "checked.pt")
    env = {**os.environ, "DCN_B200_LIB": "libdcn_b200_checked.so"}
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT, json.dumps([shapes, DTYPE]), dst], capture_output=True, text=True,
                       env=env, timeout=600)
    assert r.returncode == 0 and "ok" in r.stdout, r.stdout + r.stderr  # a range violation raises in check_status
    got = torch.load(dst)
    for name, s in SHAPES.items():
        w = gen.Workload("chk", s, DTYPE.get(name, "bf16"), seed=5, offset_dist="normal1.5_edges", bias=True)
        d = {k: (None if v is None else v.cuda()) for k, v in gen.make_inputs(w).items()}
        y = dcn.forward(d["x"], d["offset"], d["mask"], d["weight"], d["bias"], s.stride, s.pad, s.dil)
        torch.cuda.synchronize()
        dcn.check_status()
        assert torch.equal(got[name]["y"], y.cpu()), name
        # the backward sums with atomics in no fixed order: compare with the regular build's values
        gy = torch.randn(y.shape, generator=torch.Generator().manual_seed(3)).to(y.dtype).cuda()
        gx, goff, gm = dcn.backward_data(d["x"], d["offset"], d["mask"], d["weight"], gy, s.stride, s.pad, s.dil)
        gw, gb = dcn.backward_weight(d["x"], d["offset"], d["mask"], gy, tuple(d["weight"].shape), s.stride, s.pad,
                                     s.dil)
        torch.cuda.synchronize()
        for k, v in dict(gx=gx, goff=goff, gm=gm, gw=gw, gb=gb).items():
            assert_close(gen.as_f64(got[name][k]), gen.as_f64(v.cpu()), "f32", "%s %s" % (name, k))
