"""FP8 projections (section 2.4: W_V and the M W_K as one dense FP8 matmul) on
the CUDA path, against the oracle's FP8 form.

Bar: E4M3 codes and row scales bit-exact (the quantiser decides integers on
exact values); alpha, alpha*v and out at the bf16 bar (relative-L2 <= 1e-3)
against the oracle evaluated in double on the same dequantised operands.  The
bf16 oracle must be measurably further away, so the FP8 path is what ran.
"""
import numpy as np
import pytest
import torch

import oracle
from engram_cases import Problem, out_close, rel_l2, to_oracle
from hashed_gram_embedding_compress_b200 import synth

pytestmark = pytest.mark.gpu

BF16_REL = 1e-3
REDUCED = synth.SHAPES["prefill_bf16"].replace(B=2, T=700, rows_target=4099, d_hidden=512)


def _rows(rows, cols, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, cols, generator=g) * 0.02
    if rows > 3:
        x[1] = 0                    # all-zero row: scale 1, zero codes
        x[2] *= 1e4                 # scale above 1
        x[3, 5] = -3.0              # one large element, the rest in E4M3 subnormals
    return x.bfloat16()


@pytest.mark.parametrize("rows,cols", [(1, 16), (5, 48), (37, 1280), (1000, 1280), (300, 2048)])
def test_quantize_e4m3_bit_exact(rows, cols):
    p = Problem(REDUCED.replace(B=1, T=8))
    m = p.engram()
    x = _rows(rows, cols, seed=rows * 7 + cols)
    q = torch.empty((rows, cols), dtype=torch.uint8, device="cuda")
    s = torch.empty(rows, device="cuda")
    m.quantize_e4m3(x.cuda(), q, s)
    torch.cuda.synchronize()
    codes, scales = oracle.quantize_e4m3_rows(to_oracle(x))
    assert np.array_equal(q.cpu().numpy(), codes)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), scales.view(np.uint32))


def run(p: Problem, m, in_place=False, idx=None):
    sh = p.shape
    R, M, d = sh.rows_out, sh.branches, sh.d_hidden
    h = p.h.clone()
    out = h if in_place else torch.empty_like(h)
    a = torch.full((R, M), -1.0, device="cuda")
    dl = torch.full((R, M, d), float("nan"), device="cuda")
    m.forward(p.tokens.cuda(), h, out, idx=idx, t_begin=sh.t_begin, alpha=a, delta=dl)
    torch.cuda.synchronize()
    assert m.check_errors() == 0
    return out, a, dl


def check(p: Problem, rows, out, alpha, delta, in_place=False):
    _, a_ref, d_ref, o_ref = p.oracle_forward(rows, fp8=True)
    rs = torch.from_numpy(rows).cuda()
    a = alpha[rs].double().cpu().numpy()
    dl = delta[rs].double().cpu().numpy()
    o = to_oracle(out[rs])
    assert np.all((a >= 0) & (a <= 1))
    ea, ed, eo = rel_l2(a, a_ref), rel_l2(dl, d_ref), out_close(o, o_ref, "bf16")
    assert ea <= BF16_REL and ed <= BF16_REL and eo <= BF16_REL, (ea, ed, eo)
    if not in_place:  # in place, alpha v is rounded to bf16 once more before the add
        assert np.mean(o == o_ref) > 0.98
    _, _, d_bf, _ = p.oracle_forward(rows)
    assert rel_l2(dl, d_bf) > 3 * max(ed, 1e-6), "FP8 result matches the bf16 oracle instead"


def fp8_engram(p: Problem):
    m = p.engram()
    m.set_fp8(True)
    return m


def test_reduced_all_rows_ragged_and_in_place():
    # 1 400 rows (two 512-row blocks and a ragged third), 2 column tiles
    p = Problem(REDUCED)
    m = fp8_engram(p)
    out, a, dl = run(p, m)
    rows = np.arange(p.shape.rows_out)
    check(p, rows, out, a, dl)
    out2, a2, dl2 = run(p, m, in_place=True)
    assert torch.equal(dl2, dl) and torch.equal(a2, a)
    check(p, rows, out2, a2, dl2, in_place=True)
    # precomputed indices: gather, then the separate quantiser; same codes, same results
    idx = torch.empty((p.shape.rows_out, p.shape.num_tables), dtype=torch.int64, device="cuda")
    m.hash(p.tokens.cuda(), idx)
    out3, a3, dl3 = run(p, m, idx=idx)
    assert torch.equal(out3, out) and torch.equal(dl3, dl)


def test_branches_and_decode():
    # M = 2: the key launch spans the branches' columns; d = 256 is one tile per branch
    sh = REDUCED.replace(B=3, T=200, d_hidden=256, branches=2)
    p = Problem(sh)
    m = fp8_engram(p)
    out, a, dl = run(p, m)
    check(p, np.arange(sh.rows_out), out, a, dl)
    out2, a2, dl2 = run(p, m, in_place=True)
    check(p, np.arange(sh.rows_out), out2, a2, dl2, in_place=True)
    # decode: one emitted position per sequence, four branches
    shd = REDUCED.replace(B=6, T=3, t_begin=2, branches=4)
    pd = Problem(shd)
    md = fp8_engram(pd)
    out, a, dl = run(pd, md)
    check(pd, np.arange(shd.rows_out), out, a, dl)


def test_prefill_full_size_sampled():
    # the benchmarked workload and launch configuration
    p = Problem(synth.SHAPES["prefill_bf16"])
    m = fp8_engram(p)
    m.reserve(p.shape.rows_out)
    out, a, dl = run(p, m)
    check(p, p.sample_rows(64), out, a, dl)
    out2, a2, dl2 = run(p, m, in_place=True)
    assert torch.equal(dl2, dl)
    check(p, p.sample_rows(32, seed=1), out2, a2, dl2, in_place=True)


def test_short_conv_on_fp8_values():
    sh = REDUCED.replace(T=300)
    p = Problem(sh)
    m = fp8_engram(p)
    cw, nw = p.conv_weights(4)
    m.set_short_conv(cw.cuda(), nw.cuda(), 4, 3)
    out, _, dl = run(p, m)
    rows = p.sample_rows(48)
    Y, o_ref = p.oracle_forward_conv(rows, cw, nw, 3, fp8=True)
    rs = torch.from_numpy(rows).cuda()
    ey = rel_l2(dl[rs].double().cpu().numpy(), Y)
    eo = out_close(to_oracle(out[rs]), o_ref, "bf16")
    assert ey <= BF16_REL and eo <= BF16_REL, (ey, eo)


def test_switching_and_new_params():
    p = Problem(REDUCED.replace(T=200))
    m = p.engram()
    out_bf, _, dl_bf = run(p, m)
    m.set_fp8(True)
    out8, a8, dl8 = run(p, m)
    check(p, np.arange(p.shape.rows_out), out8, a8, dl8)
    m.set_fp8(False)
    out_bf2, _, dl_bf2 = run(p, m)
    assert torch.equal(out_bf2, out_bf) and torch.equal(dl_bf2, dl_bf)
    # new weights while FP8 is on are quantised again
    m.set_fp8(True)
    p.w_k_cpu = (p.w_k_cpu.float() * -0.5).bfloat16()
    p.w_k = p.w_k_cpu.cuda()
    p._w8 = None
    m.set_params(p.tables, p.w_k, p.w_v, p.norm_q, p.norm_k)
    out9, a9, dl9 = run(p, m)
    check(p, np.arange(p.shape.rows_out), out9, a9, dl9)


def test_unsupported_configurations():
    from hashed_gram_embedding_compress_b200 import engram as eg
    cases = [(synth.SHAPES["tiny_f32"], 0),                       # fp32 handle
             (REDUCED.replace(B=1, T=8, d_hidden=128), 0),         # d not a multiple of 256
             (REDUCED.replace(B=1, T=8), eg.ENGRAM_FLAG_NO_CTA_PAIRS)]
    for sh, flags in cases:
        m = Problem(sh).engram(flags=flags)
        with pytest.raises(eg.EngramError) as ei:
            m.set_fp8(True)
        assert ei.value.code == eg.ENGRAM_ERR_UNSUPPORTED
    p = Problem(REDUCED.replace(B=1, T=8))
    m = fp8_engram(p)
    e = torch.zeros((8, p.shape.d_mem), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(p.h)
    with pytest.raises(eg.EngramError) as ei:
        m.project_gate_noalloc(e, p.h, out)
    assert ei.value.code == eg.ENGRAM_ERR_UNSUPPORTED
