"""The data-parallel layer's backward (deformable_convolution_dcn_b200.data_parallel)
on one GPU, with the library's kernels: every gradient against the float64
oracle, with no process group and with a one-rank NCCL process group; the
batch blocks of a two-way split computed one after the other on this GPU and
their weight gradients summed equal the whole batch's; and an empty block
returns zeros. (A run of several ranks needs several GPUs; the two-rank
exchange itself is covered on CPU with gloo.)"""
import datetime
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from deformable_convolution_dcn_b200 import data_parallel as dp
from deformable_convolution_dcn_b200 import inputs as gen
from parity import assert_close, f64, to_dev

pytestmark = pytest.mark.gpu

# a small bfloat16 layer on the tensor-core backward kernels
SHAPE = gen.LayerShape(B=3, Cin=64, H=10, W=9, Cout=64, K=3, stride=1, pad=1)
WORK = gen.Workload("dp", SHAPE, "bf16", seed=77, offset_dist="normal1.5_edges", backward=True)
NAMES = ("grad_x", "grad_offset", "grad_mask", "grad_weight", "grad_bias")


def _oracle(host):
    a = f64(host)
    s = SHAPE
    return oracle.backward(a["x"], a["offset"], a["mask"], a["weight"], a["grad_y"], s.stride, s.pad, s.dil, s.G)


def _check_all(got, ref):
    for name, g in zip(NAMES, got):
        assert_close(g.double().cpu().numpy(), ref[name], "bf16", name)


def test_backward_without_process_group_matches_oracle():
    host = gen.make_inputs(WORK)
    d = to_dev(host)
    s = SHAPE
    got = dp.backward(d["x"], d["offset"], d["mask"], d["weight"], d["grad_y"], s.stride, s.pad, s.dil)
    torch.cuda.synchronize()
    _check_all(got, _oracle(host))


def test_backward_with_one_rank_nccl_group_matches_oracle():
    host = gen.make_inputs(WORK)
    d = to_dev(host)
    s = SHAPE
    sock = socket.socket()
    sock.bind(("127.0.0.1", 0))
    port = sock.getsockname()[1]
    sock.close()
    assert not dist.is_initialized()
    dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % port, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        got = dp.backward(d["x"], d["offset"], d["mask"], d["weight"], d["grad_y"], s.stride, s.pad, s.dil)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    _check_all(got, _oracle(host))


def test_two_blocks_sum_to_the_whole_batch():
    host = gen.make_inputs(WORK)
    d = to_dev(host)
    s = SHAPE
    ref = _oracle(host)
    gw_sum = torch.zeros((s.Cout, s.K, s.K, s.Cin), dtype=torch.float32, device="cuda")
    gb_sum = torch.zeros((s.Cout,), dtype=torch.float32, device="cuda")
    for rank in range(2):
        b0, b1 = dp.batch_shard(s.B, rank, 2)
        gx, goff, gm, gw, gb = dp.backward(d["x"][b0:b1], d["offset"][b0:b1], d["mask"][b0:b1], d["weight"],
                                           d["grad_y"][b0:b1], s.stride, s.pad, s.dil)
        torch.cuda.synchronize()
        # the per-block data gradients are the whole batch's rows of this block
        assert_close(gx.double().cpu().numpy(), ref["grad_x"][b0:b1], "bf16", "grad_x block %d" % rank)
        assert_close(goff.double().cpu().numpy(), ref["grad_offset"][b0:b1], "bf16", "grad_offset block %d" % rank)
        assert_close(gm.double().cpu().numpy(), ref["grad_mask"][b0:b1], "bf16", "grad_mask block %d" % rank)
        gw_sum += gw
        gb_sum += gb
    assert_close(gw_sum.double().cpu().numpy(), ref["grad_weight"], "bf16", "summed grad_weight")
    assert_close(gb_sum.double().cpu().numpy(), ref["grad_bias"], "bf16", "summed grad_bias")


def test_empty_block_returns_zeros():
    host = gen.make_inputs(WORK)
    d = to_dev(host)
    s = SHAPE
    e = lambda t: t[:0]
    gx, goff, gm, gw, gb = dp.backward(e(d["x"]), e(d["offset"]), e(d["mask"]), d["weight"], e(d["grad_y"]),
                                       s.stride, s.pad, s.dil)
    assert gx.shape == (0, s.H, s.W, s.Cin) and goff.shape[0] == 0 and gm.shape[0] == 0
    assert gw.shape == (s.Cout, s.K, s.K, s.Cin) and gb.shape == (s.Cout,)
    assert gw.dtype == torch.float32 and torch.count_nonzero(gw) == 0 and torch.count_nonzero(gb) == 0
    assert gw.is_cuda and gb.is_cuda
