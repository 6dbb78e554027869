"""The multi-rank host logic of bench.py on CPU: two gloo ranks.

Under torchrun every rank runs its own layer instance; the step time is the
maximum over ranks and only rank 0 prints. These tests run that reduction and
barrier logic with world_size 2 on the gloo backend (127.0.0.1), and check that
the reference arm does its work on rank 0 only.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    r, w = bench.dist_init("gloo", timeout_s=60)
    assert (r, w) == (rank, world)
    # each rank reports a different time; every rank must see the maximum
    got = bench.max_over_ranks(10.0 + 5.0 * rank)
    bench.barrier()
    env = bench.dist_env()
    dist.destroy_process_group()
    q.put((rank, got, env))


@pytest.mark.timeout(120)
def test_max_over_ranks_and_barrier_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=90) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    assert [o[1] for o in out] == [15.0, 15.0]
    assert [o[2] for o in out] == [(0, 2, 0), (1, 2, 1)]


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    bench.barrier()  # no process group: a no-op


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3", "--workload", "tiny"])
    assert capsys.readouterr().out == ""


def test_reference_arm_line_on_cpu(monkeypatch, capsys):
    """The reference arm (the float64 oracle) runs without a GPU and prints one JSON line."""
    import json
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("DCN_REFERENCE_STEP_SECONDS", "0.05")
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    bench.main(["--impl", "reference", "--steps", "2", "--warmup", "3", "--workload", "tiny"])
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "TFLOP/s"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
