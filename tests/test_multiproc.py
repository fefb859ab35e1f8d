"""N > 1 host logic on CPU: two gloo ranks.

Every rank runs its own replica of the forward (no cross-rank exchange), so the
benchmark's only collective there is the max-over-ranks of the timed region;
data-parallel training adds the sum of the dense gradients over the ranks.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    try:
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, dist, "cpu")
        seeds = bench.rank_seeds(rank)
        q.put((rank, ms, seeds["tokens"], seeds["hidden"]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_distinct_batches():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [15.0, 15.0]         # every rank sees the slowest rank's time
    assert res[0][2] != res[1][2] and res[0][3] != res[1][3]  # independent batches per rank


def _dp_worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from hashed_gram_embedding_compress_b200 import dp
    try:
        # gradients of the backward's dense outputs on each rank: dW_K, dW_V, dnorm_q, dnorm_k
        g = [torch.full((2, 3, 4), float(rank + 1)), torch.arange(12.0).reshape(3, 4) * (rank + 1),
             None, torch.full((2, 3), -1.0 - rank), torch.zeros(0)]
        dp.all_reduce_dense(g, bucket_bytes=64)   # small buckets: several collectives
        q.put((rank, [None if t is None else t.tolist() for t in g]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_sum_dense_gradients():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_dp_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for _, g in res:
        assert g[0] == torch.full((2, 3, 4), 3.0).tolist()
        assert g[1] == (torch.arange(12.0).reshape(3, 4) * 3).tolist()
        assert g[2] is None and g[3] == torch.full((2, 3), -3.0).tolist() and g[4] == []


def test_single_process_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5
