"""Row-sharded Engram tables across the GPUs of a node.

"Conditional Memory via Scalable Lookup", section 2.5 and Figure 2(a): for
training, the embedding tables are spread over the GPUs and the active rows
are exchanged.  Here row z of table s belongs to rank z % N at local row
z // N.  Every rank keeps its own shard of each table in its HBM.  The ranks
exchange the CUDA inter-process handles of their shards once (an all-gather
over torch.distributed), after which every rank holds device pointers to all
N shards of every table and hands them to the library
(Engram.set_table_shards).  The library's kernels then read a remote row with
peer loads and add a remote row's gradient with atomic adds, both over
NVLink; no step exchanges request lists or rows.

This module is host plumbing only: the split of a table into shards, the
handle exchange, and the bookkeeping of mapped pointers.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence

import torch


def shard_rows(table_rows: int, shards: int, j: int) -> int:
    """Rows of shard j: the rows z < table_rows with z % shards == j."""
    return max(0, (table_rows - j + shards - 1) // shards)


def owner_and_row(z: int, shards: int):
    """(owning shard, local row) of table row z."""
    return z % shards, z // shards


def split_table(table: torch.Tensor, shards: int) -> List[torch.Tensor]:
    """The N row shards of one table (copies, contiguous): shard j holds rows
    j, j + N, j + 2 N, ..."""
    return [table[j::shards].contiguous() for j in range(shards)]


def merge_shards(parts: Sequence[torch.Tensor]) -> torch.Tensor:
    """Inverse of split_table."""
    n = len(parts)
    rows = sum(p.shape[0] for p in parts)
    out = parts[0].new_empty((rows,) + tuple(parts[0].shape[1:]))
    for j, p in enumerate(parts):
        out[j::n] = p
    return out


class ShardSet:
    """Pointers to every shard of every table, as seen from this rank.

    own[s] is this rank's shard of table s (a device tensor).  With
    handle_fn/open_fn/close_fn left None the library's CUDA IPC entry points
    of `engram` are used; tests on hosts without a GPU pass their own."""

    def __init__(self, own: Sequence[torch.Tensor], group=None, engram=None,
                 handle_fn: Optional[Callable] = None, open_fn: Optional[Callable] = None,
                 close_fn: Optional[Callable] = None):
        import torch.distributed as dist

        self.own = list(own)
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        handle_fn = handle_fn or engram.ipc_handle
        self._open = open_fn or engram.ipc_open
        self._close = close_fn or (engram.ipc_close if engram is not None else None)
        mine = [handle_fn(t) for t in self.own]
        everyone: List = [None] * self.world
        dist.all_gather_object(everyone, mine, group=group)
        self.opened: List = []
        # ptrs[s][j]: shard j of table s
        self.ptrs = [[None] * self.world for _ in self.own]
        for j in range(self.world):
            for s, t in enumerate(self.own):
                if j == self.rank:
                    self.ptrs[s][j] = t.data_ptr() if hasattr(t, "data_ptr") else t
                else:
                    p = self._open(everyone[j][s])
                    self.opened.append(p)
                    self.ptrs[s][j] = p

    def close(self):
        """Unmap the peers' shards (after the last kernel that reads them)."""
        if self._close is not None:
            for p in self.opened:
                self._close(p)
        self.opened = []
