#!/usr/bin/env python
"""Benchmark of the DCNv2 layer on B200: forward TFLOP/s and % of roofline.

One step is one pass of the whole hot path over one batch of synthetic input:
the forward (sampling coordinates, bilinear x mask, gather, tensor-core
contraction, epilogue) and the full backward (grad_x, grad_offset, grad_mask in
one data pass; grad_weight and grad_bias in one weight pass), on the ResNet-50
conv4 3x3 DCNv2 layer (B=8, Cin=Cout=256, 50x50, K=3, stride 1, pad 1, G=1,
bfloat16 in / float32 accumulate). ``value`` is the forward's TFLOP/s (the
metric), from CUDA events around the forward launches inside the timed steps;
``ms_per_step`` covers the whole step. Inputs rotate over enough independent
sets that every step reads from HBM, not from a warm L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload conv4] [--impl ours|reference]

Multi-GPU (torchrun, one rank per GPU): every rank runs its own independent
layer instance (weak scaling, no collective on the data path); the time is the
max over ranks, the value the sum of all ranks' work over that time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "DCNv2 forward TFLOP/s and % of roofline (bf16, B200) per layer shape"
L2_BYTES = 126 * 2 ** 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks --

class ClockSampler:
    """nvidia-smi sampled every 100 ms while the timed region runs."""

    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        time.sleep(0.25)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                mx.append(float(f[1]))
                power.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(power) if power else None, "samples": len(sm), "reasons": sorted(reasons)}


# ------------------------------------------------------------ distributed --

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def dist_init(backend, timeout_s=120):
    import datetime

    import torch.distributed as dist
    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return rank, world


def max_over_ranks(value: float, device=None) -> float:
    """Max of a float over all ranks (identity with one rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# -------------------------------------------------------------- work model --

def work_model(s, elem=2, mask=True):
    """Algorithmic FLOPs and minimal HBM bytes per launch of each pass (mask=False: DCNv1, no mask tensor)."""
    nx = s.B * s.H * s.W * s.Cin
    noff = s.P * 2 * s.G * s.K * s.K
    nm = s.P * s.G * s.K * s.K if mask else 0
    nw = s.Cout * s.K * s.K * s.Cin
    ny = s.P * s.Cout
    f = s.flops()
    return {
        "forward": {"flops": f, "bytes": elem * (nx + noff + nm + nw + ny)},
        "backward_data": {"flops": f, "bytes": elem * (nx + noff + nm + nw + ny) + 4 * (nx + noff + nm)},
        "backward_weight": {"flops": f, "bytes": elem * (nx + noff + nm + ny) + 4 * (nw + s.Cout)},
    }


def roofline_entry(work, seconds, pk, sustained):
    tflop = pk["bf16_tflops_sustained" if sustained else "bf16_tflops"]
    t_flop = work["flops"] / (tflop * 1e12)
    t_hbm = work["bytes"] / (pk["hbm_gbs"] * 1e9)
    if t_flop >= t_hbm:
        ach = work["flops"] / seconds / 1e12
        return {"bound": "tensor", "achieved": round(ach, 2), "peak": tflop, "unit": "TFLOP/s",
                "frac": round(ach / tflop, 4), "roofline_frac": round(max(t_flop, t_hbm) / seconds, 4)}
    ach = work["bytes"] / seconds / 1e9
    return {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": round(ach / pk["hbm_gbs"], 4), "roofline_frac": round(max(t_flop, t_hbm) / seconds, 4)}


# ---------------------------------------------------------------- our arm --

# Device clock cycles the timed region is held for per enqueued graph replay
# (a replay with its event takes well under 50 us of host time).
HOLD_CYCLES_PER_STEP = 100_000


def run_ours(args):
    import torch

    import deformable_convolution_dcn_b200 as dcn
    from deformable_convolution_dcn_b200 import inputs as gen

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist_init("nccl")
    w = gen.WORKLOADS[args.workload]
    s = w.shape
    do_bwd = not args.forward_only
    elem = 2 if w.dtype == "bf16" else 4
    wm = work_model(s, elem, mask=w.mask_dist != "none")
    pk, pk_src = peaks()

    # rotating input sets so that every step reads its inputs from HBM
    host = gen.make_inputs(w if do_bwd else w, seed=w.seed)
    if do_bwd and "grad_y" not in host:
        g = torch.Generator().manual_seed(w.seed + 99)
        host["grad_y"] = torch.randn((s.B, s.Ho, s.Wo, s.Cout), generator=g).to(host["x"].dtype)
    set_bytes = sum(t.numel() * t.element_size() for t in host.values() if t is not None)
    out_bytes = wm["forward"]["bytes"] - elem * (s.B * s.H * s.W * s.Cin)  # rough; only sizes the rotation
    n_sets = max(2, min(64, math.ceil(3 * L2_BYTES / max(1, set_bytes + out_bytes)) + 1))
    sets = []
    for k in range(n_sets):
        d = {}
        for name, t in host.items():
            if t is None:
                d[name] = None
            else:  # every set is an independent copy in its own device memory
                d[name] = t.to(device)
        sets.append(d)
    f32 = dict(dtype=torch.float32, device=device)
    outs = []
    for k in range(n_sets):
        o = {"y": torch.empty((s.B, s.Ho, s.Wo, s.Cout), dtype=host["x"].dtype, device=device)}
        if do_bwd:
            o["grad_x"] = torch.empty((s.B, s.H, s.W, s.Cin), **f32)
            o["grad_offset"] = torch.empty(tuple(host["offset"].shape), **f32)
            o["grad_mask"] = torch.empty(tuple(host["mask"].shape), **f32) if host["mask"] is not None else None
            # grad_weight and grad_bias are views of one buffer: the data-parallel step sums it over ranks
            # with a single all-reduce
            nw = host["weight"].numel()
            o["grad_wb"] = torch.empty((nw + s.Cout,), **f32)
            o["grad_weight"] = o["grad_wb"][:nw].view(tuple(host["weight"].shape))
            o["grad_bias"] = o["grad_wb"][nw:]
        outs.append(o)
    p = dcn._params(sets[0]["x"], sets[0]["weight"], sets[0]["offset"], s.stride, s.pad, s.dil, False)
    ws = {op: (torch.empty(max(1, dcn.workspace_size(p, op)), dtype=torch.uint8, device=device))
          for op in (dcn.OP_FORWARD, dcn.OP_BACKWARD_DATA, dcn.OP_BACKWARD_WEIGHT)}

    def passes(k):
        """The three passes of one step on input set k, through the public API."""
        d, o = sets[k % n_sets], outs[k % n_sets]
        fw = lambda: dcn.forward(d["x"], d["offset"], d["mask"], d["weight"], d["bias"], s.stride, s.pad, s.dil,
                                 out=o["y"], workspace=ws[dcn.OP_FORWARD])
        bd = lambda: dcn.backward_data(d["x"], d["offset"], d["mask"], d["weight"], d["grad_y"], s.stride, s.pad,
                                       s.dil, out=(o["grad_x"], o["grad_offset"], o["grad_mask"]),
                                       workspace=ws[dcn.OP_BACKWARD_DATA])
        bw = lambda: dcn.backward_weight(d["x"], d["offset"], d["mask"], d["grad_y"], tuple(d["weight"].shape),
                                         s.stride, s.pad, s.dil, out=(o["grad_weight"], o["grad_bias"]),
                                         workspace=ws[dcn.OP_BACKWARD_WEIGHT])
        return [fw, bd, bw] if do_bwd else [fw]

    # warm up through the API, then capture each pass of each input set in a CUDA
    # graph (the library only enqueues work, so its launches capture as they are)
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        for k in range(max(args.warmup, n_sets)):
            for f in passes(k):
                f()
    torch.cuda.synchronize()
    dcn.check_status()
    graphs = []
    launches_per_step = None
    with torch.cuda.stream(stream):
        for k in range(n_sets):
            row = []
            l0 = dcn.launch_count()
            for f in passes(k):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    f()
                row.append(g)
            if launches_per_step is None:
                launches_per_step = dcn.launch_count() - l0
            graphs.append(row)
    torch.cuda.synchronize()
    npass = len(graphs[0])

    dp = args.dp and do_bwd and world > 1
    import torch.distributed as dist

    def step(k, ev=None):
        row = graphs[k % n_sets]
        for i, g in enumerate(row):
            g.replay()
            if ev is not None:
                ev[i + 1].record(stream)
        if dp:
            # data parallel: the weight gradients summed over ranks (NCCL, ordered on this stream)
            dist.all_reduce(outs[k % n_sets]["grad_wb"], op=dist.ReduceOp.SUM)
            if ev is not None:
                ev[npass + 1].record(stream)

    with torch.cuda.stream(stream):
        for k in range(args.warmup):
            step(k)
    torch.cuda.synchronize()
    dcn.check_status()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(npass + 2)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    barrier(device)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        # Hold the stream with a device-side sleep while the host enqueues every
        # timed step, so that the timed intervals hold back-to-back GPU work and
        # no host launch latency.
        torch.cuda._sleep(int(HOLD_CYCLES_PER_STEP * (args.steps * npass + 4)))
        t0.record(stream)
        for k in range(args.steps):
            evs[k][0].record(stream)
            step(args.warmup + k, evs[k])
        t1.record(stream)
    torch.cuda.synchronize()
    launches = launches_per_step * args.steps
    barrier(device)
    dcn.check_status()
    total_ms = t0.elapsed_time(t1)
    fwd_ms = [e[0].elapsed_time(e[1]) for e in evs]
    bd_ms = [e[1].elapsed_time(e[2]) for e in evs] if do_bwd else []
    bw_ms = [e[2].elapsed_time(e[3]) for e in evs] if do_bwd else []
    ar_ms = [e[npass].elapsed_time(e[npass + 1]) for e in evs] if dp else []

    total_ms_max = max_over_ranks(total_ms, device)
    fwd_sum_max = max_over_ranks(sum(fwd_ms), device)
    value = world * args.steps * wm["forward"]["flops"] / (fwd_sum_max / 1e3) / 1e12

    per = {"forward": statistics.mean(fwd_ms) / 1e3}
    if do_bwd:
        per["backward_data"] = statistics.mean(bd_ms) / 1e3
        per["backward_weight"] = statistics.mean(bw_ms) / 1e3
    # every pass is a sub-millisecond kernel timed inside a step well under a second: burst peak
    rl = {k: roofline_entry(wm[k], t, pk, sustained=False) for k, t in per.items()}
    for k in rl:
        rl[k]["traffic"] = load_traffic(args.workload, k)
        rl[k]["share_of_step"] = round(per[k] / (total_ms / args.steps / 1e3), 3)
    roof = dict(rl["forward"])
    roof.update({"kernel": "forward", "peak_source": pk_src + " (burst bf16, HBM copy)"})

    per_config = None
    if not args.no_per_config and world == 1:
        per_config = measure_per_config(args, device, pk, pk_src, rl if do_bwd else None, per)
    clk = clocks.stop()

    e2e = measure_e2e(args, s, host, device, wm) if rank == 0 else None
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, host, args.cpu_seconds)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(total_ms_max / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.description, "name": w.name, "B": s.B, "Cin": s.Cin, "Cout": s.Cout,
                       "H": s.H, "W": s.W, "K": s.K, "stride": s.stride, "pad": s.pad, "dil": s.dil, "G": s.G,
                       "step": "forward + backward_data + backward_weight" if do_bwd else "forward",
                       "l2": "inputs and outputs rotate over %d independent sets (%.0f MB each) so each step "
                             "reads from HBM" % (n_sets, (set_bytes + out_bytes) / 1e6),
                       "parallelism": "1 GPU" if world == 1 else (
                           "data parallel over %d ranks: a batch of %d per rank, grad_weight and grad_bias summed "
                           "by one NCCL all-reduce per step" % (world, s.B) if dp else
                           "%d independent replicas" % world),
                       "timing": "each pass of each input set captured once in a CUDA graph and replayed; CUDA "
                                 "events on the replay stream, which a device-side sleep holds while the host "
                                 "enqueues the timed steps",
                       "forward_path": dcn.forward_path(p)},
            "roofline": roof,
            "kernels": {k: dict(rl[k], us=round(per[k] * 1e6, 2)) for k in per},
            "forward": {"us": round(per["forward"] * 1e6, 2), "tflops": round(wm["forward"]["flops"] /
                                                                             per["forward"] / 1e12, 2),
                        "roofline_frac": rl["forward"]["roofline_frac"]},
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "clocks": clk,
        }
        if per_config is not None:
            line["per_config"] = per_config
        if dp:
            line["allreduce"] = {"us": round(statistics.mean(ar_ms) * 1e3, 2),
                                 "bytes": int(outs[0]["grad_wb"].numel() * 4)}
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()


def _source_digest(name):
    import hashlib
    try:
        return hashlib.sha256(open(os.path.join(ROOT, "deformable_convolution_dcn_b200", "csrc", name),
                                   "rb").read()).hexdigest()[:16]
    except OSError:
        return None


def load_traffic(workload, kernel, path=None):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from the
    committed ncu summary profiles/traffic.json, or None: None as well when the
    kernel's source file has changed since the counters were taken (each entry
    records the source file and its digest at capture time; a pass of several
    kernels, their sum and a list of files and digests)."""
    path = path or os.path.join(ROOT, "profiles", "traffic.json")
    try:
        e = json.load(open(path))[workload][kernel]
    except Exception:
        return None
    if isinstance(e, dict):
        # a pass of several kernels lists every source file and its digest
        srcs, shas = e.get("source", ""), e.get("sha")
        if isinstance(srcs, str):
            srcs, shas = [srcs], [shas]
        if not isinstance(shas, list) or len(shas) != len(srcs) or \
                any(h != _source_digest(f) for f, h in zip(srcs, shas)):
            return None
        return e.get("bytes")
    return None


# The layer shapes timed one by one in the default run, besides the conv4 step:
# the 224x224 RGB stem (float32; HBM-bound), the conv3 down-sampling layer and
# the conv5 dilated, grouped layer (bfloat16).
PER_CONFIG = ("stem", "conv3_s2", "conv5_d2g4", "conv4")


def time_forward(w, device, seconds, per_graph=32):
    """Forward of workload `w` alone: `per_graph` forwards over rotating input
    sets (every set evicted from L2 before it comes round again) captured in one
    CUDA graph through the public API, the graph replayed for about `seconds`
    of device time with CUDA events around every replay. Returns (seconds per
    forward, launches per forward, replays)."""
    import torch

    import deformable_convolution_dcn_b200 as dcn
    from deformable_convolution_dcn_b200 import inputs as gen
    s = w.shape
    host = gen.make_inputs(w)
    elem = host["x"].element_size()
    set_bytes = sum(t.numel() * t.element_size() for t in host.values() if t is not None) + elem * s.P * s.Cout
    n_sets = max(2, min(per_graph, math.ceil(3 * L2_BYTES / set_bytes) + 1))
    sets = [{k: (None if t is None else t.to(device)) for k, t in host.items()} for _ in range(n_sets)]
    ys = [torch.empty((s.B, s.Ho, s.Wo, s.Cout), dtype=host["x"].dtype, device=device) for _ in range(n_sets)]
    p = dcn._params(sets[0]["x"], sets[0]["weight"], sets[0]["offset"], s.stride, s.pad, s.dil, False)
    ws = torch.empty(max(1, dcn.workspace_size(p, dcn.OP_FORWARD)), dtype=torch.uint8, device=device)

    def run(k):
        d = sets[k % n_sets]
        dcn.forward(d["x"], d["offset"], d["mask"], d["weight"], d["bias"], s.stride, s.pad, s.dil,
                    out=ys[k % n_sets], workspace=ws)

    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        for k in range(n_sets + 3):
            run(k)
    torch.cuda.synchronize()
    dcn.check_status()
    g = torch.cuda.CUDAGraph()
    l0 = dcn.launch_count()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            for k in range(per_graph):
                run(k)
    launches = (dcn.launch_count() - l0) / per_graph
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
        ev[0].record(stream)
        g.replay()
        ev[1].record(stream)
    torch.cuda.synchronize()
    reps = max(3, min(4000, int(seconds / max(ev[0].elapsed_time(ev[1]) / 1e3, 1e-6))))
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
    with torch.cuda.stream(stream):
        torch.cuda._sleep(int(HOLD_CYCLES_PER_STEP * min(reps, 400)))
        for r in range(reps):
            evs[r].record(stream)
            g.replay()
        evs[reps].record(stream)
    torch.cuda.synchronize()
    dcn.check_status()
    ms = sorted(evs[r].elapsed_time(evs[r + 1]) for r in range(reps))
    del g
    return statistics.median(ms) / 1e3 / per_graph, launches, reps


def measure_per_config(args, device, pk, pk_src, step_rl, step_per):
    """Per-layer figures of the default run: each spec layer's forward timed
    alone (stem, conv3_s2, conv5_d2g4, and conv4 as a cross-check of the step),
    plus the conv4 backward passes from the timed step, each against its own
    roofline (burst bf16 peak, measured HBM copy)."""
    from deformable_convolution_dcn_b200 import inputs as gen
    out = {"peak_source": pk_src + " (burst bf16, HBM copy)",
           "timing": "per layer: 32 forwards over rotating input sets in one CUDA graph, replayed for about "
                     "%.2f s of device time; median replay / 32" % args.config_seconds}
    for name in PER_CONFIG:
        w = gen.WORKLOADS[name]
        s = w.shape
        elem = 2 if w.dtype == "bf16" else 4
        wm = work_model(s, elem, mask=w.mask_dist != "none")["forward"]
        sec, launches, reps = time_forward(w, device, args.config_seconds)
        e = roofline_entry(wm, sec, pk, sustained=False)
        e.update({"us": round(sec * 1e6, 2), "tflops": round(wm["flops"] / sec / 1e12, 2),
                  "gbs": round(wm["bytes"] / sec / 1e9, 1), "flops": wm["flops"], "bytes": wm["bytes"],
                  "dtype": w.dtype, "workload": w.description, "traffic": load_traffic(name, "forward"),
                  "launches_per_forward": launches, "replays": reps})
        out[name + "_forward"] = e
    if step_rl is not None:
        for k in ("backward_data", "backward_weight"):
            out["conv4_" + k] = dict(step_rl[k], us=round(step_per[k] * 1e6, 2))
        tot = step_per["backward_data"] + step_per["backward_weight"]
        s = gen.WORKLOADS["conv4"].shape
        out["conv4_backward"] = {"us": round(tot * 1e6, 2), "tflops": round(2 * s.flops() / tot / 1e12, 2),
                                 "frac": round(2 * s.flops() / tot / 1e12 / pk["bf16_tflops"], 4),
                                 "bound": "tensor", "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                                 "what": "backward_data + backward_weight of the conv4 step (two contractions "
                                         "of the forward's size)"}
    return out


def measure_e2e(args, s, host, device, wm):
    """Forward through the public API with host buffers: every step copies its
    inputs from pinned host memory to the device, runs the forward and reads y
    back to pinned host memory, all inside the timed region. Steps are
    pipelined over two device buffer sets on three streams, as a stream of
    requests would run: the inputs of step k+1 cross the host link while step k
    computes and step k-1's output comes back (the two directions of the link
    run concurrently)."""
    import torch

    import deformable_convolution_dcn_b200 as dcn
    # the step's inputs packed in one pinned buffer (256-byte aligned pieces), so that
    # each step's host-to-device transfer is one copy
    names = [k for k, v in host.items() if k != "grad_y" and v is not None]
    offs, total = {}, 0
    for k in names:
        offs[k] = total
        total += (host[k].numel() * host[k].element_size() + 255) // 256 * 256
    pin_buf = torch.empty(total, dtype=torch.uint8).pin_memory()
    dev_buf = [torch.empty(total, dtype=torch.uint8, device=device) for _ in range(2)]

    def view(buf, k):
        t = host[k]
        n = t.numel() * t.element_size()
        return buf[offs[k]:offs[k] + n].view(t.dtype).view(t.shape)

    for k in names:
        view(pin_buf, k).copy_(host[k])
    dev = [{k: (view(dev_buf[b], k) if k in offs else None) for k in ("x", "offset", "mask", "weight", "bias")}
           for b in range(2)]
    y_dev = [torch.empty((s.B, s.Ho, s.Wo, s.Cout), dtype=host["x"].dtype, device=device) for _ in range(2)]
    y_host = [torch.empty(y_dev[0].shape, dtype=y_dev[0].dtype).pin_memory() for _ in range(2)]
    h2d = sum(host[k].numel() * host[k].element_size() for k in names)
    d2h = y_host[0].numel() * y_host[0].element_size()
    n = max(3, min(args.steps, 20))
    s_in, s_c, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_fwd = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    started = [False, False]

    def step(k):
        b = k % 2
        with torch.cuda.stream(s_in):
            if started[b]:
                s_in.wait_event(ev_fwd[b])  # the forward of step k-2 has read this input set
            dev_buf[b].copy_(pin_buf, non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_c):
            s_c.wait_event(ev_in[b])
            if started[b]:
                s_c.wait_event(ev_out[b])  # step k-2's output has left this buffer
            d = dev[b]
            dcn.forward(d["x"], d["offset"], d["mask"], d["weight"], d["bias"], s.stride, s.pad, s.dil, out=y_dev[b])
            ev_fwd[b].record(s_c)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_fwd[b])
            y_host[b].copy_(y_dev[b], non_blocking=True)
            ev_out[b].record(s_out)
        started[b] = True

    for k in range(4):
        step(k)
    torch.cuda.synchronize()
    a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    s_c.wait_event(a)
    s_out.wait_event(a)
    for k in range(n):
        step(k)
    # the end: every stream's work of the timed steps
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_c)
    e.record(s_out)
    torch.cuda.synchronize()
    sec = a.elapsed_time(e) / 1e3 / n
    return {"value": round(wm["forward"]["flops"] / sec / 1e12, 3), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": round(sec * 1e3, 4),
            "pipelining": "inputs packed in one pinned buffer; two buffer sets, H2D / forward / D2H on three streams"}


# ---------------------------------------------------------- CPU baseline --

def _oracle_arrays(host):
    from deformable_convolution_dcn_b200 import inputs as gen
    return {k: gen.as_f64(v) for k, v in host.items()}


def cpu_baseline(w, host, seconds=10.0):
    """The float64 oracle, as it stands, on the host cores: the forward over a
    growing sample of output pixels until it runs for about `seconds`."""
    import numpy as np

    import oracle
    s = w.shape
    a = _oracle_arrays(host)
    cores = len(os.sched_getaffinity(0))
    oracle.set_threads(cores)
    # grow the pixel sample until one run takes about a tenth of the budget,
    # then repeat it until the budget is spent
    n = 64
    while True:
        pix = np.linspace(0, s.P - 1, min(n, s.P)).astype(np.int64)
        t = time.perf_counter()
        oracle.forward(a["x"], a["offset"], a["mask"], a["weight"], a["bias"], s.stride, s.pad, s.dil, s.G,
                       pixels=pix)
        dt = time.perf_counter() - t
        if dt >= seconds / 10 or len(pix) >= s.P:
            break
        n = int(n * min(8.0, max(2.0, seconds / 10 / max(dt, 1e-3))))
    reps, total = 0, 0.0
    while total < seconds:
        t = time.perf_counter()
        oracle.forward(a["x"], a["offset"], a["mask"], a["weight"], a["bias"], s.stride, s.pad, s.dil, s.G,
                       pixels=pix)
        total += time.perf_counter() - t
        reps += 1
    flops = s.flops() * len(pix) / s.P * reps
    return {"value": round(flops / total / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.max_threads(),
            "kind": "oracle", "sample": "float64 forward at %d of %d output pixels (all %d output channels), "
                                        "%d repetitions, %.1f s" % (len(pix), s.P, s.Cout, reps, total)}


# ---------------------------------------------------------- reference arm --

def run_reference(args):
    """The oracle as the reference arm: each step is the float64 forward over a
    bounded sample of the same workload's output pixels, on the host cores."""
    import numpy as np

    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle
    from deformable_convolution_dcn_b200 import inputs as gen
    w = gen.WORKLOADS[args.workload]
    s = w.shape
    host = gen.make_inputs(w)
    a = _oracle_arrays(host)
    cores = len(os.sched_getaffinity(0))
    oracle.set_threads(cores)
    budget = float(os.environ.get("DCN_REFERENCE_STEP_SECONDS", "1.0"))
    npix = 32
    while npix < s.P:   # size one step to about `budget` seconds
        pix = np.linspace(0, s.P - 1, npix).astype(np.int64)
        t = time.perf_counter()
        oracle.forward(a["x"], a["offset"], a["mask"], a["weight"], a["bias"], s.stride, s.pad, s.dil, s.G,
                       pixels=pix)
        dt = time.perf_counter() - t
        if dt >= budget / 2:
            break
        npix = min(s.P, npix * 2)
    pix = np.linspace(0, s.P - 1, npix).astype(np.int64)
    for _ in range(args.warmup):
        oracle.forward(a["x"], a["offset"], a["mask"], a["weight"], a["bias"], s.stride, s.pad, s.dil, s.G,
                       pixels=pix)
    t = time.perf_counter()
    for _ in range(args.steps):
        oracle.forward(a["x"], a["offset"], a["mask"], a["weight"], a["bias"], s.stride, s.pad, s.dil, s.G,
                       pixels=pix)
    dt = (time.perf_counter() - t) / args.steps
    flops = s.flops() * npix / s.P
    value = flops / dt / 1e12
    sample = "forward at %d of %d output pixels per step (all %d output channels)" % (npix, s.P, s.Cout)
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.description, "name": w.name, "reference": "float64 CPU oracle (oracle/)"},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "kind": "oracle",
                             "cores": oracle.max_threads(), "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_predictor(args):
    """Times the offset/mask predictor of the workload's layer (dcn_predict_offset_mask:
    a plain convolution with 3*G*K*K outputs, offsets and sigmoid masks) on its own."""
    import torch

    import deformable_convolution_dcn_b200 as dcn
    from deformable_convolution_dcn_b200 import inputs as gen

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist_init("nccl")
    w = gen.WORKLOADS[args.workload]
    s = w.shape
    elem = 2 if w.dtype == "bf16" else 4
    nc = 3 * s.G * s.K * s.K
    work = {"flops": 2.0 * s.P * nc * s.K * s.K * s.Cin,
            "bytes": elem * (s.B * s.H * s.W * s.Cin + nc * s.K * s.K * s.Cin + nc + s.P * nc)}
    pk, pk_src = peaks()
    host = gen.predictor_inputs(w.seed, s, w.dtype)
    set_bytes = sum(t.numel() * t.element_size() for t in host.values() if t is not None) + elem * s.P * nc
    n_sets = max(2, min(64, math.ceil(3 * L2_BYTES / set_bytes) + 1))
    sets = [{k: (None if t is None else t.to(device)) for k, t in host.items()} for _ in range(n_sets)]
    dt = host["x"].dtype
    outs = [(torch.empty((s.B, 2 * s.G * s.K * s.K, s.Ho, s.Wo), dtype=dt, device=device),
             torch.empty((s.B, s.G * s.K * s.K, s.Ho, s.Wo), dtype=dt, device=device)) for _ in range(n_sets)]
    p = dcn.make_params(s.B, s.H, s.W, s.Cin, 1, s.K, s.stride, s.pad, s.dil, s.G, dcn._DTYPES[dt])
    nws = dcn.predict_workspace_size(p)
    ws = torch.empty(nws, dtype=torch.uint8, device=device) if nws > 0 else None

    def run(k):
        d = sets[k % n_sets]
        dcn.predict_offset_mask(d["x"], d["w_pred"], d["b_pred"], s.K, s.stride, s.pad, s.dil, s.G,
                                workspace=ws, out=outs[k % n_sets])

    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        for k in range(max(args.warmup, n_sets)):
            run(k)
    torch.cuda.synchronize()
    dcn.check_status()
    graphs = []
    with torch.cuda.stream(stream):
        for k in range(n_sets):
            l0 = dcn.launch_count()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                run(k)
            launches_per_step = dcn.launch_count() - l0
            graphs.append(g)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for k in range(args.warmup):
            graphs[k % n_sets].replay()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    barrier(device)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        torch.cuda._sleep(int(HOLD_CYCLES_PER_STEP * (args.steps + 4)))
        t0.record(stream)
        for k in range(args.steps):
            graphs[(args.warmup + k) % n_sets].replay()
        t1.record(stream)
    torch.cuda.synchronize()
    barrier(device)
    clk = clocks.stop()
    dcn.check_status()
    ms = max_over_ranks(t0.elapsed_time(t1), device) / args.steps
    rl = roofline_entry(work, ms / 1e3, pk, sustained=False)
    rl.update({"kernel": "predictor", "traffic": load_traffic(args.workload, "predictor"),
               "peak_source": pk_src + " (burst bf16, HBM copy)"})
    if rank == 0:
        print(json.dumps({
            "metric": "DCNv2 offset/mask predictor TFLOP/s", "value": round(world * work["flops"] / ms / 1e9, 2),
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": "offset/mask predictor of: " + w.description, "outputs": nc,
                       "l2": "inputs and outputs rotate over %d independent sets" % n_sets,
                       "path": "tcgen05 implicit GEMM, sigmoid and split fused" if nws == 0 else
                               "forward kernels with zero offsets (%s), then split" % dcn.forward_path(dcn.make_params(
                                   s.B, s.H, s.W, s.Cin, (nc + 31) // 32 * 32, s.K, s.stride, s.pad, s.dil, 1,
                                   dcn._DTYPES[dt]))},
            "roofline": rl, "gpu_launches": launches_per_step * args.steps, "clocks": clk}), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()


ROI_WORKLOAD = dict(B=2, H=38, W=50, C=256, R=600, k=7, gamma=0.1, max_side=32.0)


def run_roi_pool(args):
    """Times (modulated) deformable RoI pooling, forward and backward, on a
    detector head: two 38x50x256 stride-16 maps, 300 RoIs per image, k = 7, bf16."""
    import torch

    import deformable_convolution_dcn_b200 as dcn
    from deformable_convolution_dcn_b200 import inputs as gen

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist_init("nccl")
    w = ROI_WORKLOAD
    B, H, W, C, R, k, gamma = w["B"], w["H"], w["W"], w["C"], w["R"], w["k"], w["gamma"]
    host = gen.roi_inputs(41, B, H, W, C, R, k, "bf16", max_side=w["max_side"])
    fwd_bytes = 2 * (B * H * W * C + R * 3 * k * k + R * k * k * C) + 4 * R * 5
    bwd_bytes = fwd_bytes + 4 * (B * H * W * C + R * 3 * k * k)
    set_bytes = fwd_bytes + 4 * B * H * W * C
    n_sets = max(2, min(64, math.ceil(3 * L2_BYTES / set_bytes) + 1))
    sets = [{n: (None if t is None else t.to(device)) for n, t in host.items()} for _ in range(n_sets)]
    f32 = dict(dtype=torch.float32, device=device)
    outs = [dict(y=torch.empty((R, k, k, C), dtype=torch.bfloat16, device=device), gx=torch.empty((B, H, W, C), **f32),
                 goff=torch.empty((R, 2 * k * k), **f32), gm=torch.empty((R, k * k), **f32)) for _ in range(n_sets)]
    lib = dcn._load()
    p = dcn.RoiParams(B, H, W, C, R, k, gamma, dcn.DCN_BF16, 0)
    import ctypes
    P = dcn._ptr

    def passes(i):
        d, o = sets[i % n_sets], outs[i % n_sets]
        st = dcn._stream(device)
        fw = lambda: dcn._check(lib.dcn_droi_pool_forward(ctypes.byref(p), P(d["x"]), P(d["rois"]), P(d["offset"]),
                                                          P(d["mask"]), P(o["y"]), st))
        bw = lambda: dcn._check(lib.dcn_droi_pool_backward(ctypes.byref(p), P(d["x"]), P(d["rois"]), P(d["offset"]),
                                                           P(d["mask"]), P(d["grad_y"]), P(o["gx"]), P(o["goff"]),
                                                           P(o["gm"]), st))
        return [fw, bw]

    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, n_sets)):
            for f in passes(i):
                f()
    torch.cuda.synchronize()
    dcn.check_status()
    graphs = []
    with torch.cuda.stream(stream):
        for i in range(n_sets):
            row = []
            l0 = dcn.launch_count()
            for f in passes(i):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    f()
                row.append(g)
            launches_per_step = dcn.launch_count() - l0
            graphs.append(row)
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    barrier(device)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        torch.cuda._sleep(int(HOLD_CYCLES_PER_STEP * (2 * args.steps + 4)))
        for i in range(args.steps):
            evs[i][0].record(stream)
            for j, g in enumerate(graphs[(args.warmup + i) % n_sets]):
                g.replay()
                evs[i][j + 1].record(stream)
    torch.cuda.synchronize()
    barrier(device)
    clk = clocks.stop()
    dcn.check_status()
    fwd_us = max_over_ranks(statistics.mean(e[0].elapsed_time(e[1]) for e in evs) * 1e3, device)
    bwd_us = max_over_ranks(statistics.mean(e[1].elapsed_time(e[2]) for e in evs) * 1e3, device)
    pk, pk_src = peaks()
    ach = fwd_bytes / (fwd_us * 1e-6) / 1e9
    if rank == 0:
        print(json.dumps({
            "metric": "deformable RoI pooling forward GB/s (algorithmic bytes)", "value": round(world * ach, 1),
            "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round((fwd_us + bwd_us) / 1e3, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "modulated deformable RoI pooling, two 38x50x256 maps (600x800 image at stride "
                                   "16), 300 RoIs per image with sides up to 32 feature pixels, k=7, gamma=0.1",
                       "l2": "inputs and outputs rotate over %d independent sets" % n_sets},
            "forward": {"us": round(fwd_us, 2), "bytes": fwd_bytes},
            "backward": {"us": round(bwd_us, 2), "bytes": bwd_bytes},
            "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": round(ach / pk["hbm_gbs"], 4), "traffic": None, "peak_source": pk_src},
            "gpu_launches": launches_per_step * args.steps, "clocks": clk}), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="conv4",
                    help="conv4 | conv3_s2 | conv5_d2g4 | conv4_v1 | conv4_k5 | stem | tiny | conv4_bwd")
    ap.add_argument("--forward-only", action="store_true", help="time the forward alone (not the default step)")
    ap.add_argument("--predictor", action="store_true",
                    help="time the layer's offset/mask predictor instead of the default step")
    ap.add_argument("--roi-pool", action="store_true",
                    help="time deformable RoI pooling (forward and backward) on a detector-head workload")
    ap.add_argument("--dp", action="store_true",
                    help="with several GPUs: data-parallel step (grad_weight and grad_bias all-reduced every step) "
                         "instead of independent replicas")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the per-layer forward timings (stem, conv3_s2, conv5_d2g4) of the default run")
    ap.add_argument("--config-seconds", type=float, default=0.5,
                    help="device time spent on each per-layer timing of the default run")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("at least 3 warm-up steps")
    if args.workload == "conv4_bwd":
        args.workload = "conv4"
    if args.impl == "reference":
        run_reference(args)
    elif args.predictor:
        run_predictor(args)
    elif args.roi_pool:
        run_roi_pool(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
