"""The short convolution of the module output (Eq. 5) on the CUDA path,
against the oracle: Y = SiLU(Conv1D(RMSNorm(V~))) + V~, out = h + Y.

Bars as for the rest of the forward: fp32 max-abs <= 1e-5 on Y and out;
bf16 relative-L2 <= 1e-3 on Y (fp32) and on out against the oracle's out
rounded to bf16.
"""
import numpy as np
import pytest
import torch

from engram_cases import Problem, out_close, rel_l2, to_oracle
from hashed_gram_embedding_compress_b200 import synth

pytestmark = pytest.mark.gpu

F32_TOL = 1e-5
BF16_REL = 1e-3


def run_conv(p: Problem, W=4, dil=3, in_place=False, m=None):
    sh = p.shape
    m = m or p.engram()
    cw, nw = p.conv_weights(W)
    m.set_short_conv(cw.cuda(), nw.cuda(), W, dil)
    R, M, d = sh.rows_out, sh.branches, sh.d_hidden
    h = p.h.clone()
    out = h if in_place else torch.empty_like(h)
    a = torch.full((R, M), -1.0, device="cuda")
    dl = torch.full((R, M, d), float("nan"), device="cuda")
    m.forward(p.tokens.cuda(), h, out, alpha=a, delta=dl)
    torch.cuda.synchronize()
    assert m.check_errors() == 0
    return m, out, a, dl, cw, nw


def check(p: Problem, rows, out, dl, cw, nw, dil):
    sh = p.shape
    Y, o_ref = p.oracle_forward_conv(rows, cw, nw, dil)
    rs = torch.from_numpy(rows).cuda()
    y = dl[rs].double().cpu().numpy()
    o = to_oracle(out[rs])
    if sh.dtype == "f32":
        assert np.abs(y - Y).max() <= F32_TOL
        assert out_close(o, o_ref, "f32") <= F32_TOL
    else:
        ey, eo = rel_l2(y, Y), out_close(o, o_ref, "bf16")
        assert ey <= BF16_REL and eo <= BF16_REL, (ey, eo)
        assert np.mean(o == o_ref) > 0.98


def test_f32_all_rows():
    p = Problem(synth.SHAPES["tiny_f32"])
    _, out, a, dl, cw, nw = run_conv(p)
    check(p, np.arange(p.shape.rows_out), out, dl, cw, nw, 3)


@pytest.mark.parametrize("W,dil", [(4, 3), (2, 1), (3, 4)])
def test_bf16_reduced_all_rows(W, dil):
    # 600 rows over two sequences (not a multiple of the 64-position conv tile)
    sh = synth.SHAPES["prefill_bf16"].replace(B=2, T=300, rows_target=4099, d_hidden=512)
    p = Problem(sh)
    _, out, a, dl, cw, nw = run_conv(p, W, dil)
    check(p, np.arange(sh.rows_out), out, dl, cw, nw, dil)


def test_three_branches_in_place():
    sh = synth.SHAPES["prefill_bf16"].replace(B=3, T=150, rows_target=2053, d_hidden=256, branches=3)
    p = Problem(sh)
    _, out, a, dl, cw, nw = run_conv(p, in_place=True)
    check(p, np.arange(sh.rows_out), out, dl, cw, nw, 3)


def test_full_size_sampled_in_place():
    # the benchmarked shape (32768 rows, d = 2560) and launch configuration
    p = Problem(synth.SHAPES["prefill_bf16"])
    _, out, a, dl, cw, nw = run_conv(p, in_place=True)
    check(p, p.sample_rows(40), out, dl, cw, nw, 3)


def test_zero_weights_equal_the_gated_residual_and_switching_off():
    sh = synth.SHAPES["prefill_bf16"].replace(B=2, T=333, rows_target=2053, d_hidden=256)
    p = Problem(sh)
    m = p.engram()
    ref = torch.empty_like(p.h)
    dref = torch.empty((sh.rows_out, sh.branches, sh.d_hidden), device="cuda")
    m.forward(p.tokens.cuda(), p.h, ref, delta=dref)
    d = sh.d_hidden
    m.set_short_conv(torch.zeros((d, 4), device="cuda"), torch.ones(d, device="cuda"), 4, 3)
    out = torch.empty_like(p.h)
    dl = torch.empty_like(dref)
    m.forward(p.tokens.cuda(), p.h, out, delta=dl)
    torch.cuda.synchronize()
    # Y = SiLU(0) + alpha v: the same increment, rounded the same way up to one ulp
    assert rel_l2(dl.double(), dref.double()) < 1e-6
    assert (out == ref).double().mean().item() > 0.99
    m.set_short_conv(None, None, 0, 0)
    out2 = torch.empty_like(p.h)
    m.forward(p.tokens.cuda(), p.h, out2)
    torch.cuda.synchronize()
    assert torch.equal(out2, ref)


def test_unsupported_combinations():
    from hashed_gram_embedding_compress_b200 import engram as eg
    p = Problem(synth.SHAPES["decode_mb"].replace(rows_target=1031))
    m = p.engram()
    cw, nw = p.conv_weights()
    m.set_short_conv(cw.cuda(), nw.cuda(), 4, 3)
    out = torch.empty_like(p.h)
    with pytest.raises(eg.EngramError) as ei:
        m.forward(p.tokens.cuda(), p.h, out, t_begin=p.shape.t_begin)
    assert ei.value.code == eg.ENGRAM_ERR_UNSUPPORTED
    e = torch.zeros((4, p.shape.d_mem), dtype=torch.bfloat16, device="cuda")
    h = torch.zeros((4, p.shape.branches, p.shape.d_hidden), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(eg.EngramError) as ei:
        m.project_gate_noalloc(e, h, h)
    assert ei.value.code == eg.ENGRAM_ERR_UNSUPPORTED
    for k, dil in ((5, 3), (4, 0)):
        with pytest.raises(eg.EngramError) as ei:
            m.set_short_conv(cw.cuda(), nw.cuda(), k, dil)
        assert ei.value.code == eg.ENGRAM_ERR_INVALID
