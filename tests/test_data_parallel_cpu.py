"""Host logic of the data-parallel layer on CPU: batch sharding, and the
bucketed all-reduce of the weight gradients across two gloo ranks checked
against the float64 oracle's whole-batch gradients (each rank computes its
block's gradients with the oracle, standing in for the kernels)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from deformable_convolution_dcn_b200.data_parallel import allreduce_weight_grads, batch_shard  # noqa: E402


@pytest.mark.parametrize("world", [1, 2, 3, 4, 7])
def test_batch_shard_partitions_the_batch(world):
    for B in range(0, 12):
        blocks = [batch_shard(B, r, world) for r in range(world)]
        assert blocks[0][0] == 0 and blocks[-1][1] == B
        for (a0, a1), (b0, b1) in zip(blocks, blocks[1:]):
            assert a1 == b0
        sizes = [b - a for a, b in blocks]
        assert min(sizes) >= 0 and max(sizes) - min(sizes) <= 1
        assert sizes == sorted(sizes, reverse=True)


def test_batch_shard_rejects_bad_ranks():
    with pytest.raises(ValueError):
        batch_shard(4, 2, 2)
    with pytest.raises(ValueError):
        batch_shard(4, 0, 0)


def test_single_process_is_identity():
    gw = torch.arange(6.0).reshape(2, 3)
    gb = torch.ones(2)
    out_w, out_b = allreduce_weight_grads(gw.clone(), gb.clone())
    assert torch.equal(out_w, gw) and torch.equal(out_b, gb)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import oracle
    from deformable_convolution_dcn_b200 import inputs as gen
    from deformable_convolution_dcn_b200.data_parallel import allreduce_weight_grads, batch_shard
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        s, d = gen.random_case(5, "f32", B=3, K=3, stride=1, pad=1, dil=1, G=2, Cin=4, Cout=5, H=6, W=5)
        a = {k: gen.as_f64(v) for k, v in d.items()}
        whole = oracle.backward(a["x"], a["offset"], a["mask"], a["weight"], a["grad_y"], s.stride, s.pad, s.dil,
                                s.G)
        b0, b1 = batch_shard(s.B, rank, world)
        part = oracle.backward(a["x"][b0:b1], a["offset"][b0:b1], a["mask"][b0:b1], a["weight"], a["grad_y"][b0:b1],
                               s.stride, s.pad, s.dil, s.G)
        gw = torch.from_numpy(np.ascontiguousarray(part["grad_weight"]))
        gb = torch.from_numpy(np.ascontiguousarray(part["grad_bias"]))
        allreduce_weight_grads(gw, gb)
        q.put((rank, float(np.abs(gw.numpy() - whole["grad_weight"]).max()),
               float(np.abs(gb.numpy() - whole["grad_bias"]).max()),
               float(np.abs(part["grad_x"] - whole["grad_x"][b0:b1]).max()),
               float(np.abs(gw.numpy()).max())))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_weight_gradients_summed_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=150) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for rank, ew, eb, ex, scale in out:
        assert scale > 0
        assert ew <= 1e-12 * (1 + scale), (rank, ew)
        assert eb <= 1e-12, (rank, eb)
        assert ex == 0.0, (rank, ex)
