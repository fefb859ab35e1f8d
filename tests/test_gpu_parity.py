"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bar: compressed ids and hash indices bit-exact, gathered rows bit-exact;
fp32 configs max-abs <= 1e-5 on alpha, alpha*v and out; bf16 configs
relative-L2 <= 1e-3 on alpha and alpha*v (fp32 on the device, fp64 in the
oracle) and on out against the oracle's out rounded to bf16.
"""
import numpy as np
import pytest
import torch

from engram_cases import Problem, from_bits, out_close, rel_l2, to_oracle
from hashed_gram_embedding_compress_b200 import synth

pytestmark = pytest.mark.gpu

F32_TOL = 1e-5
BF16_REL = 1e-3


def run_forward(p: Problem, m, idx=None, alpha=True, delta=True):
    sh = p.shape
    R, M, d = sh.rows_out, sh.branches, sh.d_hidden
    out = torch.empty_like(p.h)
    a = torch.full((R, M), -1.0, device="cuda") if alpha else None
    dl = torch.full((R, M, d), float("nan"), device="cuda") if delta else None
    m.forward(p.tokens.cuda(), p.h, out, idx=idx, t_begin=sh.t_begin, alpha=a, delta=dl)
    torch.cuda.synchronize()
    assert m.check_errors() == 0
    return out, a, dl


def check_indices(p: Problem, m):
    sh = p.shape
    idx = torch.empty((sh.rows_out, sh.num_tables), dtype=torch.int64, device="cuda")
    m.hash(p.tokens.cuda(), idx, t_begin=sh.t_begin)
    torch.cuda.synchronize()
    primes, mult = m.hash_params()
    assert np.array_equal(primes.numpy(), p.primes)
    assert np.array_equal(mult.numpy().view(np.uint64), p.mult)
    assert np.array_equal(idx.cpu().numpy(), p.z), "hash indices differ from the oracle"
    return idx


def check_rows(p: Problem, m, idx, rows, out, alpha, delta):
    sh = p.shape
    e_ref, a_ref, d_ref, o_ref = p.oracle_forward(rows)
    # gathered memory vectors, bit-exact
    e = torch.empty((len(rows), sh.d_mem), dtype=synth.torch_dtype(sh.dtype), device="cuda")
    m.gather(idx[torch.from_numpy(rows).cuda()].contiguous(), e)
    torch.cuda.synchronize()
    assert np.array_equal(to_oracle(e), e_ref), "gathered rows differ"
    rs = torch.from_numpy(rows).cuda()
    a = alpha[rs].double().cpu().numpy()
    dl = delta[rs].double().cpu().numpy()
    o = to_oracle(out[rs])
    assert np.all((a >= 0) & (a <= 1))
    if sh.dtype == "f32":
        assert np.abs(a - a_ref).max() <= F32_TOL
        assert np.abs(dl - d_ref).max() <= F32_TOL
        assert out_close(o, o_ref, "f32") <= F32_TOL
    else:
        ea, ed, eo = rel_l2(a, a_ref), rel_l2(dl, d_ref), out_close(o, o_ref, "bf16")
        assert ea <= BF16_REL and ed <= BF16_REL and eo <= BF16_REL, (ea, ed, eo)
        # bf16 outputs: nearly every element rounds to the same bf16 value
        assert np.mean(o == o_ref) > 0.98


def test_tiny_f32_all_rows():
    p = Problem(synth.SHAPES["tiny_f32"])
    m = p.engram()
    idx = check_indices(p, m)
    out, a, dl = run_forward(p, m)
    rows = np.arange(p.shape.rows_out)
    check_rows(p, m, idx, rows, out, a, dl)


def test_prefill_reduced_all_rows_ragged():
    # prefill structure at a size the oracle finishes in seconds: 600 rows
    # (not a multiple of the 128-row tile), several N tiles per branch
    sh = synth.SHAPES["prefill_bf16"].replace(B=2, T=300, rows_target=4099, d_hidden=512)
    p = Problem(sh)
    m = p.engram()
    idx = check_indices(p, m)
    out, a, dl = run_forward(p, m)
    check_rows(p, m, idx, np.arange(sh.rows_out), out, a, dl)


def test_prefill_full_size_sampled():
    # the benchmarked workload and launch configuration (256 x 256 tiles on CTA pairs)
    from hashed_gram_embedding_compress_b200 import engram as eg
    p = Problem(synth.SHAPES["prefill_bf16"])
    m = p.engram()
    m.reserve(p.shape.rows_out)
    idx = check_indices(p, m)
    out, a, dl = run_forward(p, m)
    check_rows(p, m, idx, p.sample_rows(96), out, a, dl)
    # without the optional outputs and with caller-supplied indices: same out
    out2, _, _ = run_forward(p, m, idx=idx, alpha=False, delta=False)
    assert torch.equal(out, out2)
    # single-CTA tiles: same bar, same values
    for flags in (eg.ENGRAM_FLAG_NO_CTA_PAIRS,):
        m1 = p.engram(flags=flags)
        out1, a1, dl1 = run_forward(p, m1)
        check_rows(p, m1, idx, p.sample_rows(32, seed=1), out1, a1, dl1)
        assert rel_l2(dl1.double(), dl.double()) < 1e-6
        check_in_place(p, m1, out1, dl1)
    check_in_place(p, m, out, dl)


def check_in_place(p: Problem, m, out, delta):
    # out aliasing h (the residual update H <- H + Y in place): the value
    # phase adds bf16(alpha v) into h, one extra rounding of alpha v
    sh = p.shape
    h2 = p.h.clone()
    a2 = torch.empty((sh.rows_out, sh.branches), device="cuda")
    d2 = torch.empty((sh.rows_out, sh.branches, sh.d_hidden), device="cuda")
    m.forward(p.tokens.cuda(), h2, h2, t_begin=sh.t_begin, alpha=a2, delta=d2)
    torch.cuda.synchronize()
    assert m.check_errors() == 0
    assert torch.equal(d2, delta)
    assert rel_l2(h2.double(), out.double()) < BF16_REL
    assert (h2 == out).double().mean().item() > 0.98
    rows = p.sample_rows(16, seed=2)
    _, _, _, o_ref = p.oracle_forward(rows)
    assert out_close(to_oracle(h2[torch.from_numpy(rows).cuda()]), o_ref, "bf16") <= BF16_REL


@pytest.mark.parametrize("shape", [
    synth.SHAPES["tiny_f32"],                                            # S = 8
    synth.SHAPES["decode_mb"],                                           # one row per block
    synth.SHAPES["tiny_f32"].replace(orders=(2, 3, 4), heads=5, T=37),    # S = 15: 17 rows per block
    synth.SHAPES["prefill_bf16"].replace(B=3, T=171, heads=3, rows_target=4099, d_hidden=256),
    # 3000 rows: 11 rows per block, so blocks straddle the sequence starts
    synth.SHAPES["prefill_bf16"].replace(B=3, T=1000, heads=3, rows_target=4099, d_hidden=256),
])
def test_fused_hash_gather_matches_separate_kernels(shape):
    # forward from tokens computes the indices on chip (one hash + gather
    # kernel); from caller-supplied indices it runs the gather kernel alone.
    # Equal memory vectors give bit-identical outputs.
    p = Problem(shape)
    m = p.engram()
    idx = check_indices(p, m)
    out1, a1, d1 = run_forward(p, m)
    out2, a2, d2 = run_forward(p, m, idx=idx)
    assert torch.equal(out1, out2) and torch.equal(a1, a2) and torch.equal(d1, d2)
    rows = np.arange(min(shape.rows_out, 64))
    check_rows(p, m, idx, rows, out1, a1, d1)


def test_decode_multibranch():
    p = Problem(synth.SHAPES["decode_mb"])
    m = p.engram()
    idx = check_indices(p, m)
    out, a, dl = run_forward(p, m)
    check_rows(p, m, idx, p.sample_rows(48), out, a, dl)


@pytest.mark.parametrize("R_B,R_T,flags", [(1, 40000, 0), (1, 20000, 0), (1, 20000, 1), (1, 10000, 0),
                                           (1, 2000, 0), (3, 5, 0), (1, 1, 0), (1, 37900, 0)])
def test_tile_widths_and_ragged_rows(R_B, R_T, flags):
    # d = 256, M = 2 lets the launcher pick CTA-pair 512 x 256 tiles (40000,
    # 37900 rows), CTA-pair 256 x 256 tiles (10000; values of 20000) or
    # single-CTA tiles (2000 and fewer; flags=1: no CTA pairs) by cost;
    # 37900 rows end in a 512-row tile whose second CTA has no rows
    sh = synth.SHAPES["prefill_bf16"].replace(B=R_B, T=R_T, rows_target=2053, d_hidden=256,
                                              branches=2)
    p = Problem(sh)
    m = p.engram(flags=flags)
    idx = check_indices(p, m)
    out, a, dl = run_forward(p, m)
    check_rows(p, m, idx, p.sample_rows(64), out, a, dl)


def test_pair_tiles_in_place():
    # 10000 rows, d = 256, M = 2: keys and values on 256 x 256 CTA-pair tiles
    # (two TMEM accumulators); in place the values are added by TMA reduce-add
    sh = synth.SHAPES["prefill_bf16"].replace(B=1, T=10000, rows_target=2053, d_hidden=256,
                                              branches=2)
    p = Problem(sh)
    m = p.engram()
    idx = check_indices(p, m)
    out, a, dl = run_forward(p, m)
    check_rows(p, m, idx, p.sample_rows(48), out, a, dl)
    check_in_place(p, m, out, dl)


@pytest.mark.parametrize("flags", [0, 1])
def test_key_tiles_do_not_straddle_branches(flags):
    # d = 384, M = 2: the key phase spans M d = 768 columns, a multiple of 256,
    # but 256-column partial-sum tiles would straddle the two branches; every
    # kernel choice must use key tiles whose width divides d
    sh = synth.SHAPES["prefill_bf16"].replace(B=2, T=9000, rows_target=2053, d_hidden=384,
                                              branches=2)
    p = Problem(sh)
    m = p.engram(flags=flags)
    idx = check_indices(p, m)
    out, a, dl = run_forward(p, m)
    check_rows(p, m, idx, p.sample_rows(64), out, a, dl)


def test_hidden_not_multiple_of_128_and_three_branches():
    sh = synth.SHAPES["decode_mb"].replace(B=37, T=9, t_begin=4, rows_target=1031, d_hidden=192,
                                           branches=3)
    p = Problem(sh)
    m = p.engram()
    idx = check_indices(p, m)
    out, a, dl = run_forward(p, m)
    check_rows(p, m, idx, np.arange(sh.rows_out), out, a, dl)


def test_f32_multibranch_and_t_begin():
    sh = synth.SHAPES["tiny_f32"].replace(B=5, T=33, t_begin=7, branches=4, d_hidden=192)
    p = Problem(sh)
    m = p.engram()
    idx = check_indices(p, m)
    out, a, dl = run_forward(p, m)
    check_rows(p, m, idx, np.arange(sh.rows_out), out, a, dl)


def test_large_hbm_sampled():
    p = Problem(synth.SHAPES["large_hbm"])
    m = p.engram()
    idx = check_indices(p, m)
    out, a, dl = run_forward(p, m, delta=False)
    rows = p.sample_rows(24)
    e_ref, a_ref, d_ref, o_ref = p.oracle_forward(rows)
    rs = torch.from_numpy(rows).cuda()
    assert rel_l2(a[rs].double().cpu(), a_ref) <= BF16_REL
    assert out_close(to_oracle(out[rs]), o_ref, "bf16") <= BF16_REL
    e = torch.empty((len(rows), p.shape.d_mem), dtype=torch.bfloat16, device="cuda")
    m.gather(idx[rs].contiguous(), e)
    assert np.array_equal(to_oracle(e), e_ref)
    # in place, four branches
    h2 = p.h.clone()
    m.forward(p.tokens.cuda(), h2, h2)
    torch.cuda.synchronize()
    assert m.check_errors() == 0
    assert rel_l2(h2.double(), out.double()) < BF16_REL
    assert out_close(to_oracle(h2[rs]), o_ref, "bf16") <= BF16_REL


def test_in_place_update_and_empty_batch():
    sh = synth.SHAPES["prefill_bf16"].replace(B=2, T=70, rows_target=3001, d_hidden=256)
    p = Problem(sh)
    m = p.engram()
    out_ref, _, _ = run_forward(p, m, alpha=False, delta=False)
    h2 = p.h.clone()
    m.forward(p.tokens.cuda(), h2, h2)  # out aliases h
    torch.cuda.synchronize()
    # in place the CTA-pair value kernels add bf16(alpha v) into h (a second
    # rounding, RN(h + RN(alpha v))); out of place every value kernel writes
    # RN(h + alpha v): equal, or one rounding step apart on a few elements
    same = (h2 == out_ref).float().mean().item()
    assert same > 0.98 and rel_l2(h2.double(), out_ref.double()) <= 1e-3
    rows = np.arange(sh.rows_out)
    _, _, _, o_ref = p.oracle_forward(rows)
    assert out_close(to_oracle(h2), o_ref, "bf16") <= 1e-3
    empty = torch.empty((0, 5), dtype=torch.int32, device="cuda")
    m.forward(empty, h2[:0], h2[:0])
    m.hash(empty, torch.empty((0, sh.num_tables), dtype=torch.int64, device="cuda"))
    assert m.check_errors() == 0


def test_out_of_range_tokens_are_reported_not_read():
    from hashed_gram_embedding_compress_b200 import engram as eg
    sh = synth.SHAPES["tiny_f32"]
    p = Problem(sh)
    m = p.engram()
    bad = p.tokens.clone()
    bad[0, 5] = sh.vocab + 7
    bad[1, 0] = -3
    idx = torch.empty((sh.rows_out, sh.num_tables), dtype=torch.int64, device="cuda")
    m.hash(bad.cuda(), idx)
    assert m.check_errors() == eg.ENGRAM_ERR_BOUNDS
    assert m.check_errors() == 0  # the error word is cleared by reading it
    # rows whose n-grams avoid the bad positions are unaffected
    good = idx.cpu().numpy().reshape(sh.B, sh.T, -1)
    ref = p.z.reshape(sh.B, sh.T, -1)
    assert np.array_equal(good[0, :5], ref[0, :5]) and np.array_equal(good[0, 8:], ref[0, 8:])
    # indices outside a table: zero rows, flagged
    idx[3, 2] = int(p.primes[2]) + 5
    e = torch.ones((sh.rows_out, sh.d_mem), device="cuda")
    m.gather(idx, e)
    assert m.check_errors() == eg.ENGRAM_ERR_BOUNDS
    assert torch.all(e[3, 2 * sh.d_head:3 * sh.d_head] == 0)


def test_bounded_wait_expiry_is_reported_and_context_survives():
    # a kernel waits on an mbarrier nothing arrives at, another on a count in
    # global memory that never reaches its target (the one-launch short-call
    # kernel's wait): each bounded wait expires (2 s), each timeout is
    # reported, and the next forward is exact
    from hashed_gram_embedding_compress_b200 import engram as eg
    sh = synth.SHAPES["tiny_f32"]
    p = Problem(sh)
    m = p.engram()
    assert m.selftest_timeout() == eg.ENGRAM_ERR_TIMEOUT
    assert m.check_errors() == 0
    idx = check_indices(p, m)
    out, a, dl = run_forward(p, m)
    check_rows(p, m, idx, np.arange(sh.rows_out), out, a, dl)
