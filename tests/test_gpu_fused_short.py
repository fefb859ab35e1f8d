"""Short calls (at most 256 rows, bf16, d a multiple of 256, M <= 4) run steps
5-7 in one launch: key clusters store their partial sums and count themselves
done, value clusters wait for the count, form alpha and write out = h + alpha v.

Parity with the oracle on every row of ragged short calls, and against the
separate key, alpha and value launches (ENGRAM_FLAG_NO_FUSED_SHORT): on the
decode workload, whose separate key launch uses the same 256 x 256 pair tiles,
alpha bit-identical (the same partial sums added in the same order); out and
alpha v within the bf16 bar.  Consecutive calls, CUDA graph replays and chained
in-place updates check the counters and the order of h's reads and writes."""
import numpy as np
import pytest
import torch

from engram_cases import Problem, out_close, rel_l2, to_oracle
from hashed_gram_embedding_compress_b200 import engram as eg
from hashed_gram_embedding_compress_b200 import synth

pytestmark = pytest.mark.gpu

BF16_REL = 1e-3


def _forward(p: Problem, m, h=None, out=None):
    sh = p.shape
    R, M, d = sh.rows_out, sh.branches, sh.d_hidden
    h = p.h if h is None else h
    out = torch.empty_like(h) if out is None else out
    a = torch.full((R, M), -1.0, device="cuda")
    dl = torch.full((R, M, d), float("nan"), device="cuda")
    n0 = m.kernel_launches()
    m.forward(p.tokens.cuda(), h, out, t_begin=sh.t_begin, alpha=a, delta=dl)
    torch.cuda.synchronize()
    assert m.check_errors() == 0
    return out, a, dl, m.kernel_launches() - n0


def _check_oracle(p: Problem, rows, out, a, dl):
    _, a_ref, d_ref, o_ref = p.oracle_forward(rows)
    rs = torch.from_numpy(rows).cuda()
    ea = rel_l2(a[rs].double().cpu().numpy(), a_ref)
    ed = rel_l2(dl[rs].double().cpu().numpy(), d_ref)
    eo = out_close(to_oracle(out[rs]), o_ref, "bf16")
    assert ea <= BF16_REL and ed <= BF16_REL and eo <= BF16_REL, (ea, ed, eo)
    assert np.mean(to_oracle(out[rs]) == o_ref) > 0.98


@pytest.mark.parametrize("B,T,t_begin,M,d", [
    (256, 3, 2, 4, 256),   # 256 rows: both CTAs of every pair hold rows
    (200, 3, 2, 3, 512),   # ragged second half
    (129, 1, 0, 2, 256),   # one row in the second half
    (128, 2, 1, 1, 768),   # the second half empty
    (37, 9, 8, 4, 256),    # few rows, four branches
    (1, 1, 0, 1, 256),     # one row
])
def test_short_calls_every_row_against_oracle_and_separate_launches(B, T, t_begin, M, d):
    sh = synth.SHAPES["decode_mb"].replace(B=B, T=T, t_begin=t_begin, branches=M, d_hidden=d,
                                           rows_target=1031)
    p = Problem(sh)
    m = p.engram()
    out, a, dl, launches = _forward(p, m)
    assert launches == 2  # hash + gather, then steps 5-7
    _check_oracle(p, np.arange(sh.rows_out), out, a, dl)
    # the separate launches (their key tiles may differ: equal up to fp32 order)
    m3 = p.engram(flags=eg.ENGRAM_FLAG_NO_FUSED_SHORT)
    out3, a3, dl3, launches3 = _forward(p, m3)
    assert launches3 == 4
    assert rel_l2(a.double(), a3.double()) < 1e-6
    assert rel_l2(dl.double(), dl3.double()) < 1e-6
    assert (out == out3).double().mean().item() > 0.99


def test_decode_workload_in_place_and_out_of_place():
    p = Problem(synth.SHAPES["decode_mb"])
    sh = p.shape
    m = p.engram()
    out, a, dl, launches = _forward(p, m)
    assert launches == 2
    _check_oracle(p, p.sample_rows(64), out, a, dl)
    # in place (out aliases h): the same values as out of place, rounded once
    h2 = p.h.clone()
    _, a2, dl2, _ = _forward(p, m, h=h2, out=h2)
    assert torch.equal(a2, a) and torch.equal(dl2, dl) and torch.equal(h2, out)
    # the separate launches key on the same 256 x 256 pair tiles: the same
    # partial sums, added in the same order, give the same alpha
    m3 = p.engram(flags=eg.ENGRAM_FLAG_NO_FUSED_SHORT)
    out3, a3, dl3, launches3 = _forward(p, m3)
    assert launches3 == 4
    assert torch.equal(a, a3)
    assert rel_l2(dl.double(), dl3.double()) < 1e-6
    assert (out == out3).double().mean().item() > 0.99


def test_consecutive_calls_and_graph_replays_start_from_zero_counters():
    sh = synth.SHAPES["decode_mb"].replace(rows_target=1031, d_hidden=512)
    p = Problem(sh)
    m = p.engram()
    ref, a_ref, _, _ = _forward(p, m)
    # back-to-back calls on one stream, no synchronisation between them
    outs = [torch.empty_like(p.h) for _ in range(6)]
    for o in outs:
        m.forward(p.tokens.cuda(), p.h, o, t_begin=sh.t_begin)
    torch.cuda.synchronize()
    assert m.check_errors() == 0
    for o in outs:
        assert torch.equal(o, ref)
    # replays of a captured call
    tok = p.tokens.cuda()
    out_g = torch.empty_like(p.h)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        m.forward(tok, p.h, out_g, t_begin=sh.t_begin)
    for _ in range(4):
        out_g.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert m.check_errors() == 0
        assert torch.equal(out_g, ref)
    del g


def test_in_place_steps_match_repeated_out_of_place_updates():
    """Three in-place decode updates h <- h + alpha v equal three out-of-place
    calls chained through fresh buffers (each step reads the previous step's
    output, which the launch before the gather wrote)."""
    sh = synth.SHAPES["decode_mb"].replace(rows_target=1031, d_hidden=512, branches=2)
    p = Problem(sh)
    m = p.engram()
    h_in = p.h.clone()
    for _ in range(3):
        m.forward(p.tokens.cuda(), h_in, h_in, t_begin=sh.t_begin)
    cur = p.h.clone()
    for _ in range(3):
        nxt = torch.empty_like(cur)
        m.forward(p.tokens.cuda(), cur, nxt, t_begin=sh.t_begin)
        cur = nxt
    torch.cuda.synchronize()
    assert m.check_errors() == 0
    assert torch.equal(h_in, cur)


@pytest.mark.parametrize("B,T,t_begin,M,d,flags,launches", [
    (257, 3, 2, 2, 256, 0, 4),    # 257 rows: more than one 256-row block
    (64, 3, 2, 2, 384, 0, 4),     # d not a multiple of 256
    (64, 3, 2, 2, 256, 2, 4),     # ENGRAM_FLAG_NO_FUSED_SHORT
    (64, 3, 2, 2, 256, 1, 4),     # ENGRAM_FLAG_NO_CTA_PAIRS
    (256, 3, 2, 4, 512, 0, 2),    # taken
])
def test_which_calls_take_the_one_launch_path(B, T, t_begin, M, d, flags, launches):
    sh = synth.SHAPES["decode_mb"].replace(B=B, T=T, t_begin=t_begin, branches=M, d_hidden=d,
                                           rows_target=1031)
    p = Problem(sh)
    m = p.engram(flags=flags)
    out, a, dl, n = _forward(p, m)
    assert n == launches
    _check_oracle(p, p.sample_rows(48), out, a, dl)
