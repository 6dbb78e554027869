"""Host logic of bench.py without a GPU: the algorithmic work model the
roofline fractions divide by, the bound classification, the peaks and the
committed traffic figures it reads, and its argument checks."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from deformable_convolution_dcn_b200 import inputs as gen  # noqa: E402


def test_conv4_work_model_matches_hand_count():
    s = gen.WORKLOADS["conv4"].shape
    wm = bench.work_model(s, elem=2)
    # 2 * M * N * K with M = 8*50*50 pixels, N = 256 outputs, K = 9 * 256
    assert wm["forward"]["flops"] == 2 * 20000 * 256 * 2304
    # x 10.24 MB + offset 0.72 MB + mask 0.36 MB + weight 1.18 MB + y 10.24 MB (bf16)
    assert wm["forward"]["bytes"] == 2 * (8 * 50 * 50 * 256 + 20000 * 18 + 20000 * 9 + 256 * 9 * 256 + 20000 * 256)
    # the backward passes read the same tensors and write float32 gradients
    assert wm["backward_data"]["bytes"] > wm["forward"]["bytes"]
    assert wm["backward_weight"]["flops"] == wm["forward"]["flops"]


def test_dcnv1_work_model_drops_the_mask():
    s = gen.WORKLOADS["conv4_v1"].shape
    with_mask = bench.work_model(s, 2, mask=True)["forward"]["bytes"]
    without = bench.work_model(s, 2, mask=False)["forward"]["bytes"]
    assert with_mask - without == 2 * 20000 * 9


def test_roofline_entry_picks_the_binding_resource():
    pk = {"hbm_gbs": 6500.0, "bf16_tflops": 1650.0, "bf16_tflops_sustained": 1370.0}
    # conv4: 23.6 GFLOP vs 22.7 MB -> tensor-bound
    conv4 = bench.work_model(gen.WORKLOADS["conv4"].shape, 2)["forward"]
    e = bench.roofline_entry(conv4, 60e-6, pk, sustained=True)
    assert e["bound"] == "tensor" and e["unit"] == "TFLOP/s" and e["peak"] == 1370.0
    assert e["achieved"] == pytest.approx(conv4["flops"] / 60e-6 / 1e12, rel=1e-3)
    assert e["frac"] == pytest.approx(e["achieved"] / 1370.0, rel=1e-3)
    # the float32 stem: 0.17 GFLOP vs 18.9 MB -> HBM-bound
    stem = bench.work_model(gen.WORKLOADS["stem"].shape, 4)["forward"]
    e = bench.roofline_entry(stem, 16e-6, pk, sustained=False)
    assert e["bound"] == "hbm" and e["unit"] == "GB/s"
    assert e["achieved"] == pytest.approx(stem["bytes"] / 16e-6 / 1e9, rel=1e-3)
    assert 0 < e["roofline_frac"] <= 1


def test_peaks_come_from_the_measured_file_when_present():
    pk, src = bench.peaks()
    assert set(pk) == {"hbm_gbs", "bf16_tflops", "bf16_tflops_sustained"}
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    assert src == ("measured" if os.path.exists(path) else "fallback")
    assert all(v > 0 for v in pk.values())


def test_committed_traffic_figures_are_read():
    d = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    for wl, kernels in d.items():
        if wl.startswith("_"):
            continue
        for k, v in kernels.items():
            assert v["bytes"] > 0
            srcs = v["source"] if isinstance(v["source"], list) else [v["source"]]
            shas = v["sha"] if isinstance(v["sha"], list) else [v["sha"]]
            for f in srcs:
                assert os.path.exists(os.path.join(ROOT, "deformable_convolution_dcn_b200", "csrc", f))
            if "kernels" in v:  # a pass of several kernels: their sum
                assert sum(v["kernels"].values()) == v["bytes"]
            # a figure is reported only while its kernels' sources are the ones it was taken on
            fresh = all(h == bench._source_digest(f) for f, h in zip(srcs, shas))
            assert bench.load_traffic(wl, k) == (v["bytes"] if fresh else None)
    assert bench.load_traffic("conv4", "no_such_kernel") is None


def test_traffic_of_a_changed_kernel_is_dropped(tmp_path):
    p = tmp_path / "traffic.json"
    good = bench._source_digest("fwd_tc.cu")
    p.write_text(json.dumps({"conv4": {"forward": {"bytes": 123, "source": "fwd_tc.cu", "sha": good},
                                       "backward_data": {"bytes": 456, "source": "fwd_tc.cu", "sha": "0" * 16}}}))
    assert bench.load_traffic("conv4", "forward", path=str(p)) == 123
    assert bench.load_traffic("conv4", "backward_data", path=str(p)) is None
    # a pass of several kernels: every listed source must be unchanged
    other = bench._source_digest("bwd_data_tc.cu")
    p.write_text(json.dumps({"conv4": {
        "backward_data": {"bytes": 7, "source": ["fwd_tc.cu", "bwd_data_tc.cu"], "sha": [good, other]},
        "backward_weight": {"bytes": 8, "source": ["fwd_tc.cu", "bwd_data_tc.cu"], "sha": [good, "0" * 16]}}}))
    assert bench.load_traffic("conv4", "backward_data", path=str(p)) == 7
    assert bench.load_traffic("conv4", "backward_weight", path=str(p)) is None


def test_arguments_are_checked():
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])  # at least three warm-up steps
    with pytest.raises(SystemExit):
        bench.main(["--impl", "other"])
