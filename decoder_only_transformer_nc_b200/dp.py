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


def _bucket_layout(tensors: dict):
    """[(key, shape, offset)] of every gradient view of the bucket, and the
    body's length in floats (each view padded to 4 floats: 16 bytes)."""
    shapes = [("wte", tensors["wte"].shape), ("lm_head", tensors["lm_head"].shape)]
    for l, lw in enumerate(tensors["layers"]):
        shapes += [((l, n), lw[n].shape) for n in NAMES]
    ex = tensors.get("extras") or {}
    for k, v in ex.items():  # per-layer lists keep their None entries
        if isinstance(v, list):
            shapes += [(("extras", k, l), x.shape) for l, x in enumerate(v) if x is not None]
        elif v is not None:
            shapes.append((("extras", k), v.shape))
    out, off = [], 0
    for key, shp in shapes:
        n = 1
        for d in shp:
            n *= d
        out.append((key, shp, off))
        off += (n + 3) // 4 * 4
    return out, off


def grad_bucket(tensors: dict, device=None):
    """One flat fp32 buffer holding a gradient for every weight of ``tensors``
    (the layout of ``Model.tensors``, the further terms' "extras" included),
    each view starting on a 16-byte boundary, plus a last slot for the local
    target count.  Returns (flat, grads) with ``grads`` in the layout
    ``forward_backward`` takes; the buffer is zeroed."""
    layout, body = _bucket_layout(tensors)
    ex = tensors.get("extras") or {}
    dev = device if device is not None else tensors["wte"].device
    flat = torch.zeros(body + 4, dtype=torch.float32, device=dev)
    grads = {"layers": [dict() for _ in tensors["layers"]]}
    if ex:
        grads["extras"] = {k: ([None] * len(v) if isinstance(v, list) else None) for k, v in ex.items()}
    for key, shp, o in layout:
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


def bucket_slices(tensors: dict):
    """[(name, start, stop)]: the bucket of ``grad_bucket(tensors)`` cut into
    the pieces the training step's backward finishes one after another, in
    that order -- "lm_head" (right after the logit gradient), "layer l" for
    l = L-1 .. 0 (a layer's six gradients are adjacent), "wte" (the embedding
    backward comes last), and "tail": the further terms' gradients, written
    before the embedding backward, followed by the count slot.  Together they
    cover the whole buffer once."""
    layout, body = _bucket_layout(tensors)
    off = {key: o for key, _, o in layout}
    L = len(tensors["layers"])
    starts = [off[(l, NAMES[0])] for l in range(L)]
    ends = starts[1:] + [min([o for key, _, o in layout if isinstance(key, tuple) and key[0] == "extras"],
                             default=body)]
    out = [("lm_head", off["lm_head"], starts[0] if L else body)]
    out += [(f"layer {l}", starts[l], ends[l]) for l in reversed(range(L))]
    out.append(("wte", 0, off["lm_head"]))
    out.append(("tail", ends[-1] if L else body, body + 4))
    return out


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


def average_grads_sliced_(flat: torch.Tensor, slices, local_count: float, group=None, before=None) -> torch.Tensor:
    """``average_grads_`` one slice at a time (``bucket_slices`` order): each
    slice is scaled by the local count and all-reduced on its own, the count
    slot travelling with the last one, then the body is divided by the global
    count.  ``before(k)``, when given, runs ahead of slice k (the overlapped
    schedule makes the side stream wait there).  Every rank must pass the same
    slices in the same order."""
    if not slices or slices[-1][2] != flat.numel():
        raise ValueError("the last slice must end with the bucket's count slot")
    for k, (_, a, b) in enumerate(slices):
        if before is not None:
            before(k)
        piece = flat[a:b]
        if b == flat.numel():  # the slice with the count slot
            flat[a:b - 4].mul_(float(local_count))
            flat[-4:].zero_()
            flat[-4] = float(local_count)
        else:
            piece.mul_(float(local_count))
        dist.all_reduce(piece, op=dist.ReduceOp.SUM, group=group)
    flat[:-4].div_(flat[-4].clamp_min(1.0))
    return flat


def backward_finish_entries(kinds, n_layer: int):
    """For each of ``bucket_slices``' pieces, the index of the traced launch
    after which it is final, from the kinds of one traced training step
    (``LaunchTrace.kinds()``): lm_head after the first weight-gradient product
    that follows the logit gradient; layer L-1-k after the backward's k-th
    "emb_bwd" launch (the QKV weight-gradient scatter, the layer's last
    gradient write); wte and the tail after the last "emb_bwd" (the embedding
    backward, which follows every untraced kernel of the further terms)."""
    try:
        ce = kinds.index("ce_bwd")
        lm = kinds.index("gemm_wgrad", ce)
    except ValueError:
        raise ValueError("the trace holds no training step's backward") from None
    emb = [i for i in range(ce, len(kinds)) if kinds[i] == "emb_bwd"]
    if len(emb) != n_layer + 1:
        raise ValueError(f"expected {n_layer + 1} emb_bwd launches in the backward, found {len(emb)}")
    return [lm] + emb[:n_layer] + [emb[-1], emb[-1]]


class OverlappedGradAverage:
    """The data-parallel gradient average of the training step, overlapped
    with its backward: each piece of the bucket (``bucket_slices``) is
    all-reduced on a side stream as soon as the traced launch that finishes it
    has run, so the NCCL transfers of layers L-1 .. 1 run under the backward
    of the layers below them.  ``launch`` goes right after
    ``forward_backward(..., trace=trace)`` has been enqueued on ``stream``; on
    return ``stream`` waits for the average."""

    def __init__(self, tensors: dict, flat: torch.Tensor, group=None):
        self.flat, self.group = flat, group
        self.slices = bucket_slices(tensors)
        self.n_layer = len(tensors["layers"])
        self.comm = torch.cuda.Stream(device=flat.device)

    def launch(self, trace, local_count: float, stream=None):
        from . import _check, lib
        stream = stream if stream is not None else torch.cuda.current_stream(self.flat.device)
        entries = backward_finish_entries(trace.kinds(), self.n_layer)
        comm = self.comm

        def before(k):
            _check(lib().nc_stream_wait_event(comm.cuda_stream, trace.end_event(entries[k])),
                   "nc_stream_wait_event")

        # (no wait for the whole stream here: each slice waits for its own launch)
        with torch.cuda.stream(comm):
            average_grads_sliced_(self.flat, self.slices, local_count, self.group, before)
        stream.wait_stream(comm)
        return self.flat
