"""Data-parallel plumbing of the forward (one process per GPU).

The forward shards by batch row ("从文本到聊天模型" §4.5: each rank reads its own
rows): every rank holds the whole model and runs ``nc_forward`` on its own
[B, T] shard.  The only exchange is the global mean loss: each rank
contributes (local mean * local count, local count) and one all-reduce of that
2-vector (fp64) gives sum / count over all ranks' non-ignored targets.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_seed(base_seed: int, rank: int) -> int:
    """Seed of rank `rank`'s token shard (distinct rows on every rank)."""
    return base_seed + rank


def reduce_loss_into(buf: torch.Tensor, local_mean: torch.Tensor, local_count: float, group=None):
    """All-reduce (local_mean * local_count, local_count) into `buf` (2 x fp64,
    preallocated on the loss's device) and return the global mean (a view).
    A rank with no valid targets passes local_count = 0 (its mean is ignored)."""
    if local_count > 0:
        buf[0] = local_mean.double() * local_count
    else:
        buf[0] = 0.0
    buf[1] = float(local_count)
    dist.all_reduce(buf, op=dist.ReduceOp.SUM, group=group)
    return buf[0] / buf[1]


def global_mean_loss(local_mean: torch.Tensor, local_count: float, group=None) -> torch.Tensor:
    buf = torch.zeros(2, dtype=torch.float64, device=local_mean.device)
    return reduce_loss_into(buf, local_mean, local_count, group)
