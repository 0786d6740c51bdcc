"""Data-parallel plumbing of multi-GPU runs (one process per GPU, torch.distributed).

Every (image, window, head) unit of the attention is independent, so a
data-parallel run gives each rank its own images and needs no exchange in the
attention itself.  theta is one parameter shared by all images, so its
gradient is the sum of the ranks' gradients: the one collective of the path
(48 floats at Swin-T stage 1).  Times are taken as the maximum over ranks.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from .inputs import make_inputs


def rank_inputs(B: int, H: int, W: int, heads: int, d: int, rank: int, device, qk_scale: float = 1.0,
                with_dout: bool = True) -> dict:
    """This rank's images (distinct per rank) and the shared theta."""
    return make_inputs(B, H, W, heads, d, device=device, qk_scale=qk_scale, with_dout=with_dout, shard=rank)


def allreduce_dtheta(dtheta: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the ranks' dtheta in place (no-op without an initialised process group)."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(dtheta, op=dist.ReduceOp.SUM, group=group)
    return dtheta


def allreduce_param_grads(*grads, group=None):
    """Sum each rank's gradients of parameters shared by the whole batch (theta,
    the low-rank bias factors) in place."""
    for g in grads:
        if g is not None:
            allreduce_dtheta(g, group)
    return grads


def max_over_ranks(value: float, device, group=None) -> float:
    """The largest value over all ranks (the job's time is its slowest rank's)."""
    if not (dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1):
        return float(value)
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
