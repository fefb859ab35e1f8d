"""Host-resident tables: deterministic prefetch over PCIe (section 2.5, Fig. 2b).

The prefetch hashes the tokens ahead, de-duplicates the addressed rows, copies
each distinct row once from pinned host memory into an HBM staging buffer
(host threads + copy engines, or zero-copy loads on a few CTAs), and the
forward gathers from there.  Its results must equal the device-resident path
bit for bit (same rows, same kernels after the gather), whichever route moved
the rows.
"""
import numpy as np
import pytest
import torch

from engram_cases import Problem, out_close, rel_l2, to_oracle
from hashed_gram_embedding_compress_b200 import synth

pytestmark = pytest.mark.gpu


def _pair(shape):
    host = Problem(shape.replace(table_location="pinned_host"))
    dev_tables = [t.cuda() for t in host.tables]
    return host, dev_tables


ROUTES = [("host_threads", 0), ("host_threads", 1), ("zero_copy", 16), ("zero_copy", 0)]


@pytest.mark.parametrize("route", ROUTES)
def test_prefetch_then_forward_equals_device_tables(route):
    from hashed_gram_embedding_compress_b200 import engram as eg
    sh = synth.SHAPES["prefill_bf16"].replace(B=2, T=1500, rows_target=1 << 18)
    p, dev_tables = _pair(sh)
    assert p.tables[0].is_pinned()
    m = p.engram()
    m.set_prefetch(*route)
    # reference: the same inputs with device-resident tables
    md = eg.Engram(eg.make_config(vocab=sh.vocab, cvocab=sh.cvocab, comp_map=p.comp_map,
                                  orders=sh.orders, heads=sh.heads, d_head=sh.d_head,
                                  d_hidden=sh.d_hidden, branches=sh.branches, dtype=sh.dtype,
                                  table_rows_target=sh.rows_target, hash_seed=p.hash_seed))
    md.set_params(dev_tables, p.w_k, p.w_v, p.norm_q, p.norm_k)
    tok = p.tokens.cuda()
    ref = torch.empty_like(p.h)
    a_ref = torch.empty((sh.rows_out, 1), device="cuda")
    md.forward(tok, p.h, ref, alpha=a_ref)

    side = torch.cuda.Stream()
    n = m.prefetch(tok, stream=side, want_count=True)
    # distinct (table, row) pairs among the oracle's indices
    want = sum(len(np.unique(p.z[:, s])) for s in range(sh.num_tables))
    assert n == want
    out = torch.empty_like(p.h)
    alpha = torch.empty((sh.rows_out, 1), device="cuda")
    m.forward(tok, p.h, out, alpha=alpha)  # waits for the prefetch on the side stream
    torch.cuda.synchronize()
    assert m.check_errors() == 0
    assert torch.equal(out, ref) and torch.equal(alpha, a_ref)
    rows = p.sample_rows(24)
    _, a_o, _, o_o = p.oracle_forward(rows)
    rs = torch.from_numpy(rows).cuda()
    assert rel_l2(alpha[rs].double().cpu(), a_o) <= 1e-3
    assert out_close(to_oracle(out[rs]), o_o, "bf16") <= 1e-3


@pytest.mark.parametrize("route", ROUTES[::2])
def test_double_buffered_prefetch_and_call_order(route):
    from hashed_gram_embedding_compress_b200 import engram as eg
    sh = synth.SHAPES["prefill_bf16"].replace(B=2, T=300, rows_target=1 << 16, d_hidden=256)
    p, dev_tables = _pair(sh)
    m = p.engram()
    m.set_prefetch(*route)
    tok_a = p.tokens.cuda()
    tok_b = torch.flip(p.tokens, dims=[1]).contiguous().cuda()
    with pytest.raises(eg.EngramError) as ei:
        m.forward(tok_a, p.h, torch.empty_like(p.h))
    assert ei.value.code == eg.ENGRAM_ERR_STATE
    side = torch.cuda.Stream()
    m.prefetch(tok_a, stream=side)
    m.prefetch(tok_b, stream=side)
    with pytest.raises(eg.EngramError) as ei:
        m.prefetch(tok_a, stream=side)  # a third pending prefetch has no staging slot
    assert ei.value.code == eg.ENGRAM_ERR_STATE
    md = eg.Engram(eg.make_config(vocab=sh.vocab, cvocab=sh.cvocab, comp_map=p.comp_map,
                                  orders=sh.orders, heads=sh.heads, d_head=sh.d_head,
                                  d_hidden=sh.d_hidden, branches=sh.branches, dtype=sh.dtype,
                                  table_rows_target=sh.rows_target, hash_seed=p.hash_seed))
    md.set_params(dev_tables, p.w_k, p.w_v, p.norm_q, p.norm_k)
    for tok in (tok_a, tok_b):  # consumed in prefetch order
        out, ref = torch.empty_like(p.h), torch.empty_like(p.h)
        m.forward(tok, p.h, out)
        md.forward(tok, p.h, ref)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    assert m.check_errors() == 0


def _expected_hits(p, calib_z, step_z, max_rows):
    """Hot rows: the max_rows (table, row) keys the calibration indices address
    most often (ties: lower table, then lower row); hits: the step's distinct
    keys among them.  Computed from the oracle's indices alone."""
    S = calib_z.shape[1]
    keys = (np.arange(S, dtype=np.int64)[None, :] << 40) | calib_z
    uk, cnt = np.unique(keys.ravel(), return_counts=True)
    order = np.lexsort((uk, -cnt))  # count descending, then key ascending
    hot = set(uk[order[:max_rows]].tolist())
    step = np.unique(((np.arange(S, dtype=np.int64)[None, :] << 40) | step_z).ravel())
    return sum(1 for k in step.tolist() if k in hot)


@pytest.mark.parametrize("max_rows,route", [(1000, ROUTES[0]), (10 ** 7, ROUTES[0]),
                                            (1000, ROUTES[2])])
def test_hot_row_cache_serves_rows_and_keeps_results(max_rows, route):
    from hashed_gram_embedding_compress_b200 import engram as eg
    import oracle
    sh = synth.SHAPES["prefill_bf16"].replace(B=2, T=1200, rows_target=1 << 17, d_hidden=256)
    p, _ = _pair(sh)
    m0 = p.engram()
    m1 = p.engram()
    m1.set_prefetch(*route)
    side = torch.cuda.Stream()
    # calibrate on other tokens of the same distribution (the step's own
    # indices would overstate the hits)
    calib = synth.make_tokens(sh, synth.stream_seeds(sh, extra=7))
    m1.build_hot_cache(calib.cuda(), max_rows)
    tok = p.tokens.cuda()
    outs = []
    for m in (m0, m1):
        m.prefetch(tok, stream=side)
        out = torch.empty_like(p.h)
        m.forward(tok, p.h, out)
        torch.cuda.synchronize()
        assert m.check_errors() == 0
        outs.append(out)
    assert torch.equal(outs[0], outs[1])  # the cached rows are the same bytes
    _, calib_z, _, _ = oracle.forward_indices(calib.numpy(), p.comp_map.numpy(), sh.cvocab,
                                              sh.orders, sh.heads, p.hash_seed, sh.rows_target)
    want = _expected_hits(p, calib_z, p.z, max_rows)
    assert m1.prefetch_hot_hits() == want and want > 0
    assert m0.prefetch_hot_hits() == 0


def test_hot_row_cache_needs_host_tables():
    from hashed_gram_embedding_compress_b200 import engram as eg
    p = Problem(synth.SHAPES["tiny_f32"])
    m = p.engram()
    with pytest.raises(eg.EngramError) as ei:
        m.build_hot_cache(p.tokens.cuda(), 10)
    assert ei.value.code == eg.ENGRAM_ERR_STATE


def test_set_prefetch_rejects_bad_modes_and_pending_prefetches():
    from hashed_gram_embedding_compress_b200 import engram as eg
    sh = synth.SHAPES["prefill_bf16"].replace(B=1, T=64, rows_target=1031, d_hidden=256)
    p, _ = _pair(sh)
    m = p.engram()
    with pytest.raises(eg.EngramError) as ei:
        m._check(eg.lib.engram_set_prefetch(m._h, 7, 0))
    assert ei.value.code == eg.ENGRAM_ERR_INVALID
    side = torch.cuda.Stream()
    tok = p.tokens.cuda()
    with pytest.raises(eg.EngramError) as ei:
        m.prefetch_wait()  # nothing pending
    assert ei.value.code == eg.ENGRAM_ERR_STATE
    m.prefetch(tok, stream=side)
    with pytest.raises(eg.EngramError) as ei:
        m.set_prefetch("zero_copy")
    assert ei.value.code == eg.ENGRAM_ERR_STATE
    m.prefetch_wait()
    m.forward(tok, p.h, torch.empty_like(p.h))
    m.set_prefetch("zero_copy")
    d = Problem(synth.SHAPES["tiny_f32"]).engram()
    with pytest.raises(eg.EngramError) as ei:
        d.set_prefetch("host_threads")
    assert ei.value.code == eg.ENGRAM_ERR_STATE


def test_offload_workload_shapes_against_the_oracle():
    """The host-offloaded workload's own shapes: B = 4 x T = 8192 tokens,
    vocab 128000 -> 98560, 16 host tables of 160-byte rows (primes >= 2^21
    here, 5.4 GB pinned, instead of the benchmark's 100 GB), M = 4 branches of
    d = 4096.  Two steps run the benchmark's pipeline (the next step's
    prefetch issued before the current forward) with the host-thread route;
    every index is checked against the oracle's distinct-row count, alpha and
    out against the oracle on sampled rows, and the zero-copy route must give
    the same bytes."""
    from hashed_gram_embedding_compress_b200 import engram as eg
    sh = synth.SHAPES["offload"].replace(rows_target=1 << 21)
    p = Problem(sh)
    assert p.tables[0].is_pinned() and sh.branches == 4 and sh.d_hidden == 4096
    tok = [p.tokens.cuda(), torch.flip(p.tokens, dims=[1]).contiguous().cuda()]
    side = torch.cuda.Stream()
    outs = {}
    for route in (("host_threads", 0), ("zero_copy", 0)):
        m = p.engram()
        m.set_prefetch(*route)
        m.reserve(sh.rows_out)
        n0 = m.prefetch(tok[0], stream=side, want_count=True)
        want = sum(len(np.unique(p.z[:, s])) for s in range(sh.num_tables))
        assert n0 == want
        res = []
        for k in range(2):
            if k + 1 < len(tok):
                m.prefetch(tok[k + 1], stream=side)  # next step's rows, overlapped
            out = torch.empty_like(p.h)
            alpha = torch.empty((sh.rows_out, sh.branches), device="cuda")
            m.forward(tok[k], p.h, out, alpha=alpha)
            res.append((out, alpha))
        torch.cuda.synchronize()
        assert m.check_errors() == 0
        outs[route[0]] = res
    for (o1, a1), (o2, a2) in zip(outs["host_threads"], outs["zero_copy"]):
        assert torch.equal(o1, o2) and torch.equal(a1, a2)
    out, alpha = outs["host_threads"][0]
    rows = p.sample_rows(24)
    _, a_o, _, o_o = p.oracle_forward(rows)
    rs = torch.from_numpy(rows).cuda()
    assert rel_l2(alpha[rs].double().cpu(), a_o) <= 1e-3
    assert out_close(to_oracle(out[rs]), o_o, "bf16") <= 1e-3
    # the second step (reversed sequences) against a device-table forward of the same tokens
    md = eg.Engram(eg.make_config(vocab=sh.vocab, cvocab=sh.cvocab, comp_map=p.comp_map,
                                  orders=sh.orders, heads=sh.heads, d_head=sh.d_head,
                                  d_hidden=sh.d_hidden, branches=sh.branches, dtype=sh.dtype,
                                  table_rows_target=sh.rows_target, hash_seed=p.hash_seed))
    md.set_params([t.cuda() for t in p.tables], p.w_k, p.w_v, p.norm_q, p.norm_k)
    ref = torch.empty_like(p.h)
    md.forward(tok[1], p.h, ref)
    torch.cuda.synchronize()
    assert torch.equal(outs["host_threads"][1][0], ref)


@pytest.mark.parametrize("route", ROUTES[::2])
def test_prefetch_then_short_multibranch_call(route):
    """A decode-sized call (256 rows, four branches) on host tables: the rows
    come through the prefetch staging, then keys, alpha and values run in one
    launch; results equal the device-resident tables' bit for bit, in place."""
    from hashed_gram_embedding_compress_b200 import engram as eg
    sh = synth.SHAPES["decode_mb"].replace(rows_target=1 << 16, d_hidden=512)
    p, dev_tables = _pair(sh)
    m = p.engram()
    m.set_prefetch(*route)
    md = eg.Engram(eg.make_config(vocab=sh.vocab, cvocab=sh.cvocab, comp_map=p.comp_map,
                                  orders=sh.orders, heads=sh.heads, d_head=sh.d_head,
                                  d_hidden=sh.d_hidden, branches=sh.branches, dtype=sh.dtype,
                                  table_rows_target=sh.rows_target, hash_seed=p.hash_seed))
    md.set_params(dev_tables, p.w_k, p.w_v, p.norm_q, p.norm_k)
    tok = p.tokens.cuda()
    R, M = sh.rows_out, sh.branches
    ref = p.h.clone()
    a_ref = torch.empty((R, M), device="cuda")
    n0 = md.kernel_launches()
    md.forward(tok, ref, ref, t_begin=sh.t_begin, alpha=a_ref)
    assert md.kernel_launches() - n0 == 2  # the gather, then the one-launch projections

    side = torch.cuda.Stream()
    m.prefetch(tok, t_begin=sh.t_begin, stream=side)
    out = p.h.clone()
    alpha = torch.empty((R, M), device="cuda")
    m.forward(tok, out, out, t_begin=sh.t_begin, alpha=alpha)
    torch.cuda.synchronize()
    assert m.check_errors() == 0 and md.check_errors() == 0
    assert torch.equal(out, ref) and torch.equal(alpha, a_ref)
    rows = p.sample_rows(32)
    _, a_o, _, o_o = p.oracle_forward(rows)
    rs = torch.from_numpy(rows).cuda()
    assert rel_l2(alpha[rs].double().cpu(), a_o) <= 1e-3
    assert out_close(to_oracle(out[rs]), o_o, "bf16") <= 1e-3
