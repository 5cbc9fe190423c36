"""Data-parallel plumbing (one process per GPU).

The batch shards by row ("从文本到聊天模型" §4.5: each rank reads its own rows):
every rank holds the whole model and runs the library on its own [B, T] shard.

* Forward: the only exchange is the global mean loss.  Each rank contributes
  (local mean * local count, local count); one all-reduce of that 2-vector
  (fp64) gives sum / count over all ranks' non-ignored targets.
* Training micro-step (``nc_forward_backward``): each rank's gradients are of
  its local mean loss.  The gradient of the global mean is
  sum_r count_r g_r / sum_r count_r.  All weight gradients live in one flat
  fp32 bucket (``grad_bucket``) whose last slot carries the count, so one
  all-reduce of count * g, followed by a device-side division, averages them
  with no host synchronisation (``average_grads_``).
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


NAMES = ("c_q", "c_k", "c_v", "attn_proj", "c_fc", "mlp_proj")


def grad_bucket(tensors: dict, device=None):
    """One flat fp32 buffer holding a gradient for every weight of ``tensors``
    (the layout of ``Model.tensors``, the further terms' "extras" included),
    each view starting on a 16-byte boundary, plus a last slot for the local
    target count.  Returns (flat, grads) with ``grads`` in the layout
    ``forward_backward`` takes; the buffer is zeroed."""
    shapes = [("wte", tensors["wte"].shape), ("lm_head", tensors["lm_head"].shape)]
    for l, lw in enumerate(tensors["layers"]):
        shapes += [((l, n), lw[n].shape) for n in NAMES]
    ex = tensors.get("extras") or {}
    for k, v in ex.items():  # per-layer lists keep their None entries
        if isinstance(v, list):
            shapes += [(("extras", k, l), x.shape) for l, x in enumerate(v) if x is not None]
        elif v is not None:
            shapes.append((("extras", k), v.shape))
    offs, off = [], 0
    for _, shp in shapes:
        offs.append(off)
        n = 1
        for d in shp:
            n *= d
        off += (n + 3) // 4 * 4
    dev = device if device is not None else tensors["wte"].device
    flat = torch.zeros(off + 4, dtype=torch.float32, device=dev)
    grads = {"layers": [dict() for _ in tensors["layers"]]}
    if ex:
        grads["extras"] = {k: ([None] * len(v) if isinstance(v, list) else None) for k, v in ex.items()}
    for (key, shp), o in zip(shapes, offs):
        n = 1
        for d in shp:
            n *= d
        view = flat[o:o + n].view(shp)
        if isinstance(key, tuple) and key[0] == "extras":
            if len(key) == 3:
                grads["extras"][key[1]][key[2]] = view
            else:
                grads["extras"][key[1]] = view
        elif isinstance(key, tuple):
            grads["layers"][key[0]][key[1]] = view
        else:
            grads[key] = view
    return flat, grads


def average_grads_(flat: torch.Tensor, local_count: float, group=None) -> torch.Tensor:
    """In place: the bucket's gradients (of each rank's local mean loss) become
    the gradient of the global mean loss over every rank's counted targets."""
    body = flat[:-4]
    body.mul_(float(local_count))
    flat[-4:].zero_()
    flat[-4] = float(local_count)
    dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    body.div_(flat[-4].clamp_min(1.0))
    return flat
