"""Row-sharded table layout on CPU: row z of table s lives in shard z % N at
local row z // N ("Conditional Memory via Scalable Lookup", section 2.5,
Figure 2a: the training layout spreads the tables over the GPUs)."""
import numpy as np
import torch

import oracle
from hashed_gram_embedding_compress_b200 import shards, synth


def test_split_merge_and_owner_mapping_against_the_oracle_gather():
    sh = synth.SHAPES["tiny_f32"]
    seeds = synth.stream_seeds(sh)
    primes = oracle.table_primes(sh.rows_target, sh.num_tables)
    tables = synth.make_tables([int(p) for p in primes], sh.d_head, sh.dtype, seeds)
    _, z, _, _ = oracle.forward_indices(synth.make_tokens(sh, seeds).numpy(),
                                        synth.make_comp_map(sh, seeds).numpy(), sh.cvocab,
                                        sh.orders, sh.heads, synth.make_hash_seed(seeds),
                                        sh.rows_target)
    e_ref = oracle.gather([t.numpy() for t in tables], z)
    for N in (1, 2, 3, 8):
        parts = [shards.split_table(t, N) for t in tables]
        for s, t in enumerate(tables):
            assert [p.shape[0] for p in parts[s]] == [shards.shard_rows(t.shape[0], N, j)
                                                      for j in range(N)]
            assert sum(p.shape[0] for p in parts[s]) == t.shape[0]
            assert torch.equal(shards.merge_shards(parts[s]), t)
        e = np.empty_like(e_ref)
        for r in range(z.shape[0]):
            for s in range(z.shape[1]):
                o, loc = shards.owner_and_row(int(z[r, s]), N)
                e[r, s * sh.d_head:(s + 1) * sh.d_head] = parts[s][o][loc].numpy()
        assert np.array_equal(e, e_ref)


def test_shard_rows_edge_cases():
    assert [shards.shard_rows(10, 4, j) for j in range(4)] == [3, 3, 2, 2]
    assert [shards.shard_rows(3, 4, j) for j in range(4)] == [1, 1, 1, 0]
    assert shards.owner_and_row(13, 4) == (1, 3)
