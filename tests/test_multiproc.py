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


def _shard_worker(rank, world, port, q):
    """One rank of a row-sharded table set: it keeps shard `rank` of every
    table, exchanges (stand-in) handles of its shards, and resolves every
    (table, shard) to the right owner.  The data exchange stands in for the
    peer loads: the shards' contents are all-gathered and every row the
    oracle gathers is read through (owner, local row); the row gradients of
    both ranks' lookups are summed into the owners' shards."""
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import numpy as np

    import oracle
    from hashed_gram_embedding_compress_b200 import shards, synth
    try:
        sh = synth.SHAPES["tiny_f32"]
        seeds = synth.stream_seeds(sh)
        primes = oracle.table_primes(sh.rows_target, sh.num_tables)
        tables = synth.make_tables([int(p) for p in primes], sh.d_head, sh.dtype, seeds)
        own = [shards.split_table(t, world)[rank] for t in tables]
        for s, t in enumerate(own):
            assert t.shape[0] == shards.shard_rows(int(primes[s]), world, rank)
        # stand-in handles: (rank, table) tags; "opening" one yields the tag
        ss = shards.ShardSet(own, handle_fn=lambda t, r=rank, o=own: (r, [x is t for x in o].index(True)),
                             open_fn=lambda hnd: ("peer",) + tuple(hnd))
        layout = [[ss.ptrs[s][j] if j != rank else ("own", s) for j in range(world)]
                  for s in range(len(own))]
        # data: every rank's shards, then the oracle's gather of this rank's tokens
        parts = []
        for s, t in enumerate(own):
            # shard sizes differ by at most one row: pad to shard 0's
            n = shards.shard_rows(int(primes[s]), world, 0)
            buf = torch.zeros((n, t.shape[1]))
            buf[:t.shape[0]] = t
            bufs = [torch.zeros_like(buf) for _ in range(world)]
            dist.all_gather(bufs, buf)
            parts.append(bufs)
        tok = synth.make_tokens(sh, synth.stream_seeds(sh, extra=rank))
        _, z, _, _ = oracle.forward_indices(tok.numpy(), synth.make_comp_map(sh, seeds).numpy(),
                                            sh.cvocab, sh.orders, sh.heads,
                                            synth.make_hash_seed(seeds), sh.rows_target)
        e_ref = oracle.gather([t.numpy() for t in tables], z)
        e = np.empty_like(e_ref)
        for r in range(z.shape[0]):
            for s in range(z.shape[1]):
                o, loc = shards.owner_and_row(int(z[r, s]), world)
                e[r, s * sh.d_head:(s + 1) * sh.d_head] = parts[s][o][loc].numpy()
        # gradients: each rank's row gradients land in the owners' shards
        de = np.random.default_rng(rank).standard_normal(e_ref.shape)
        full = oracle.table_grad(de, z, [int(p) for p in primes], sh.d_head)
        tot = [torch.from_numpy(np.array(g, copy=True)) for g in full]
        for t in tot:
            dist.all_reduce(t)
        mine = [t[rank::world].numpy() for t in tot]
        q.put((rank, layout, bool(np.array_equal(e, e_ref)),
               [m.tolist() for m in mine[:2]], [g.tolist() for g in full[:2]]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_row_sharded_tables():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    import numpy as np
    for rank, layout, gathered_ok, mine, _ in res:
        assert gathered_ok  # every looked-up row read through (owner, local row) is the table's
        for s, row in enumerate(layout):
            for j, entry in enumerate(row):
                # shard j of table s resolves to rank j's handle for table s
                assert entry == (("own", s) if j == rank else ("peer", j, s))
    # the owners' gradient shards together are the sum of both ranks' scatters
    for s in range(2):
        total = np.array(res[0][4][s]) + np.array(res[1][4][s])
        assert np.allclose(np.array(res[0][3][s]), total[0::2])
        assert np.allclose(np.array(res[1][3][s]), total[1::2])
