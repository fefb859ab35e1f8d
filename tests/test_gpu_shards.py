"""Row-sharded tables on one GPU ("Conditional Memory via Scalable Lookup",
section 2.5, Figure 2a: the training layout spreads the tables over GPUs).

Row z of table s lives in shard z % N at local row z // N.  Here the N
shards of every table sit in this GPU's memory, so the kernels' addressing of
the owner's shard is checked end to end; only the NVLink transport (the same
kernels with peers' pointers) is not exercised.  The forward must equal the
unsharded one bit for bit; the backward's table gradients, written into the
owners' gradient shards, must merge into the unsharded gradients.
"""
import numpy as np
import pytest
import torch

from engram_cases import Problem, rel_l2
from hashed_gram_embedding_compress_b200 import shards, synth

pytestmark = pytest.mark.gpu

SHAPE = synth.SHAPES["prefill_bf16"].replace(B=2, T=300, rows_target=4099, d_hidden=512)


def _sharded(p: Problem, N: int):
    parts = [shards.split_table(t, N) for t in p.tables]
    m = p.engram()
    m.set_table_shards(parts)
    return m, parts


@pytest.mark.parametrize("N", [1, 2, 3, 8])
def test_sharded_forward_equals_whole_tables(N):
    p = Problem(SHAPE)
    ref_m = p.engram()
    tok = p.tokens.cuda()
    ref = torch.empty_like(p.h)
    a_ref = torch.empty((SHAPE.rows_out, 1), device="cuda")
    ref_m.forward(tok, p.h, ref, alpha=a_ref)
    m, parts = _sharded(p, N)
    out = torch.empty_like(p.h)
    alpha = torch.empty_like(a_ref)
    m.forward(tok, p.h, out, alpha=alpha)  # fused hash + gather
    # the gather from given indices
    idx = torch.empty((SHAPE.rows_out, SHAPE.num_tables), dtype=torch.int64, device="cuda")
    m.hash(tok, idx)
    e = torch.empty((SHAPE.rows_out, SHAPE.d_mem), dtype=torch.bfloat16, device="cuda")
    m.gather(idx, e)
    e_ref = torch.empty_like(e)
    ref_m.gather(idx, e_ref)
    torch.cuda.synchronize()
    assert m.check_errors() == 0
    assert torch.equal(out, ref) and torch.equal(alpha, a_ref)
    assert torch.equal(e, e_ref)
    # the oracle's rows, read through (owner, local row)
    rows = np.arange(0, SHAPE.rows_out, 37)
    z = p.z[rows]
    got = e[torch.from_numpy(rows).cuda()].cpu()
    for i in range(len(rows)):
        for s in range(SHAPE.num_tables):
            o, loc = shards.owner_and_row(int(z[i, s]), N)
            assert torch.equal(got[i, s * SHAPE.d_head:(s + 1) * SHAPE.d_head], parts[s][o][loc].cpu())


def test_sharded_fp8_forward_equals_whole_tables():
    p = Problem(SHAPE)
    ref_m = p.engram()
    ref_m.set_fp8(True)
    tok = p.tokens.cuda()
    ref = torch.empty_like(p.h)
    ref_m.forward(tok, p.h, ref)
    m, _ = _sharded(p, 4)
    m.set_fp8(True)
    out = torch.empty_like(p.h)
    m.forward(tok, p.h, out)
    torch.cuda.synchronize()
    assert m.check_errors() == 0 and torch.equal(out, ref)


def test_sharded_backward_scatters_into_the_owners_shards():
    p = Problem(SHAPE)
    sh = p.shape
    M, d, dm, N = sh.branches, sh.d_hidden, sh.d_mem, 3
    dout = synth.make_grad_out(sh, p.seeds, device="cuda")
    tok = p.tokens.cuda()

    def grads(shard_rows=None):
        g = dict(dw_k=torch.zeros((M, d, dm), device="cuda"),
                 dw_v=torch.zeros((d, dm), device="cuda"),
                 dnorm_q=torch.zeros((M, d), device="cuda"),
                 dnorm_k=torch.zeros((M, d), device="cuda"))
        if shard_rows is None:
            g["dtables"] = [torch.zeros((int(pr), sh.d_head), device="cuda") for pr in p.primes]
        else:
            g["dtables"] = [torch.zeros((n, sh.d_head), device="cuda") for n in shard_rows]
        return g

    ref_m = p.engram()
    g0 = grads()
    dh0 = torch.empty_like(p.h)
    ref_m.backward(tok, p.h, dout, dh0, **g0)
    m, parts = _sharded(p, N)
    rows = [shards.shard_rows(int(pr), N, j) for pr in p.primes for j in range(N)]
    g1 = grads(rows)
    dh1 = torch.empty_like(p.h)
    m.backward(tok, p.h, dout, dh1, **g1)
    torch.cuda.synchronize()
    assert m.check_errors() == 0
    assert torch.equal(dh1, dh0)
    for k in ("dw_k", "dw_v", "dnorm_q", "dnorm_k"):
        assert rel_l2(g1[k].double(), g0[k].double()) < 1e-6, k
    for s in range(sh.num_tables):
        merged = shards.merge_shards(g1["dtables"][s * N:(s + 1) * N])
        assert merged.shape == g0["dtables"][s].shape
        assert rel_l2(merged.double(), g0["dtables"][s].double()) < 1e-6
        assert merged.abs().max() > 0


def test_set_table_shards_rejects_bad_input():
    from hashed_gram_embedding_compress_b200 import engram as eg
    p = Problem(SHAPE)
    m = p.engram()
    parts = [shards.split_table(t, 2) for t in p.tables]
    with pytest.raises(eg.EngramError) as ei:
        m.set_table_shards([[t.cpu() for t in row] for row in parts])  # host memory
    assert ei.value.code == eg.ENGRAM_ERR_INVALID
    with pytest.raises(eg.EngramError) as ei:
        m.set_table_shards([row * 5 for row in parts])  # 10 shards > ENGRAM_MAX_SHARDS
    assert ei.value.code == eg.ENGRAM_ERR_INVALID
