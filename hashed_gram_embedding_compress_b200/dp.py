"""Data-parallel training plumbing: the gradient exchange after engram_backward.

Each rank runs the backward on its own batch; the dense gradients (W_K, W_V and
the RMSNorm weights) are then summed over the ranks with one all-reduce per
bucket of same-dtype tensors (NCCL between GPUs; any torch.distributed backend
works).  The table gradients are not reduced here: they are dense per-table
arrays touched in few rows, for which an exchange of the touched rows (or
row-sharded tables) is the right collective.
"""
from __future__ import annotations

from typing import Iterable, Optional

import torch


def all_reduce_dense(grads: Iterable[Optional[torch.Tensor]], group=None,
                     bucket_bytes: int = 64 << 20) -> None:
    """Sum every tensor of `grads` (None entries skipped) over the ranks of
    `group`, in place.  Tensors are packed into buckets of at most
    bucket_bytes (a larger tensor forms its own bucket) so that few
    collectives are issued.  No-op without an initialised process group or
    with one rank."""
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return
    bucket: list = []
    state = {"bytes": 0}

    def flush():
        if not bucket:
            return
        flat = torch.cat([t.reshape(-1) for t in bucket])
        dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
        off = 0
        for t in bucket:
            n = t.numel()
            t.copy_(flat[off:off + n].view_as(t))
            off += n
        bucket.clear()
        state["bytes"] = 0

    for t in grads:
        if t is None or t.numel() == 0:
            continue
        nb = t.numel() * t.element_size()
        if bucket and (t.dtype != bucket[0].dtype or t.device != bucket[0].device or
                       state["bytes"] + nb > bucket_bytes):
            flush()
        bucket.append(t)
        state["bytes"] += nb
    flush()
