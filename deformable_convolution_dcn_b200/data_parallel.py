"""Data-parallel DCNv2 layer across ranks: one process per GPU, the batch split
by ranks, and one summed all-reduce of the weight gradients per step.

The layer's output pixels are independent in the forward, and in the backward
every gradient but grad_weight and grad_bias stays with the pixels (and input
rows) of its own batch entries. So the batch is sharded in contiguous blocks,
each rank runs the layer's kernels on its block, and the only exchange is the
sum over ranks of grad_weight [Cout, K, K, Cin] and grad_bias [Cout] (2.36 MB
in float32 for the ResNet-50 conv4 layer), sent as one bucket so that the
collective is a single launch. With torch.distributed on the NCCL backend the
all-reduce runs over NVLink / NVSwitch, ordered after the backward on the
caller's current stream; any backend works for the host logic.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def batch_shard(B: int, rank: int, world: int) -> tuple[int, int]:
    """[start, stop) of this rank's contiguous block of the batch: sizes differ
    by at most one, the first B % world ranks taking the extra entry; ranks
    beyond B get an empty block."""
    if B < 0 or world < 1 or not 0 <= rank < world:
        raise ValueError("need B >= 0 and 0 <= rank < world (got B=%d rank=%d world=%d)" % (B, rank, world))
    q, r = divmod(B, world)
    start = rank * q + min(rank, r)
    return start, start + q + (1 if rank < r else 0)


def allreduce_weight_grads(grad_weight: torch.Tensor, grad_bias: torch.Tensor | None = None, group=None):
    """Sums grad_weight (and grad_bias) over the ranks of `group` in place, as
    one bucket. A no-op without an initialised process group of more than one rank."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return grad_weight, grad_bias
    parts = [grad_weight] + ([grad_bias] if grad_bias is not None else [])
    if len(parts) == 1 and grad_weight.is_contiguous():
        dist.all_reduce(grad_weight, op=dist.ReduceOp.SUM, group=group)
        return grad_weight, grad_bias
    bucket = torch.cat([t.reshape(-1) for t in parts])
    dist.all_reduce(bucket, op=dist.ReduceOp.SUM, group=group)
    o = 0
    for t in parts:
        n = t.numel()
        t.copy_(bucket[o:o + n].view_as(t))
        o += n
    return grad_weight, grad_bias


def backward(x, offset, mask, weight, grad_y, stride=1, padding=0, dilation=1, *, group=None, need_bias=True):
    """Backward of this rank's batch block (x, offset, mask, grad_y hold only
    that block) with the weight gradients summed over all ranks.

    Returns grad_x, grad_offset, grad_mask (this block's, float32) and
    grad_weight, grad_bias (the whole batch's, float32, identical on every rank).
    """
    from deformable_convolution_dcn_b200 import backward_data, backward_weight
    if x.shape[0] == 0:
        # an empty block still joins the collective, with zero weight gradients
        f32 = dict(dtype=torch.float32, device=x.device)
        gw = torch.zeros(tuple(weight.shape), **f32)
        gb = torch.zeros((weight.shape[0],), **f32) if need_bias else None
        allreduce_weight_grads(gw, gb, group)
        return (torch.zeros(tuple(x.shape), **f32), torch.zeros(tuple(offset.shape), **f32),
                None if mask is None else torch.zeros(tuple(mask.shape), **f32), gw, gb)
    gx, goff, gm = backward_data(x, offset, mask, weight, grad_y, stride, padding, dilation,
                                 need_mask=mask is not None)
    gw, gb = backward_weight(x, offset, mask, grad_y, tuple(weight.shape), stride, padding, dilation,
                             need_bias=need_bias)
    allreduce_weight_grads(gw, gb, group)
    return gx, goff, gm, gw, gb
