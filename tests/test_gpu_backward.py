"""Backward of the lookup-and-gate step (training) on the CUDA path, against
the oracle's exact derivative of the forward.

Bar: fp32 handles max-abs <= 1e-5 x max(1, max |reference|) on every
gradient; bf16 handles relative-L2 <= 1e-3, with dk and dv rounded to bf16 on
both sides before the weight and table GEMMs (what the library does for bf16
operands), and dh compared after rounding the oracle's dh to bf16.
"""
import numpy as np
import pytest
import torch

import oracle
from engram_cases import Problem, rel_l2, to_oracle
from hashed_gram_embedding_compress_b200 import synth

pytestmark = pytest.mark.gpu

BF16_REL = 1e-3
F32_TOL = 1e-5
REDUCED = synth.SHAPES["prefill_bf16"].replace(B=2, T=300, rows_target=4099, d_hidden=512)


def run_backward(p: Problem, m, dout, idx=None, tables=True, grads=None):
    sh = p.shape
    M, d, dm = sh.branches, sh.d_hidden, sh.d_mem
    g = grads or dict(
        dw_k=torch.zeros((M, d, dm), device="cuda"), dw_v=torch.zeros((d, dm), device="cuda"),
        dnorm_q=torch.zeros((M, d), device="cuda"), dnorm_k=torch.zeros((M, d), device="cuda"),
        dtables=[torch.zeros((int(pr), sh.d_head), device="cuda") for pr in p.primes]
        if tables else None)
    dh = torch.full_like(p.h, float("nan"))
    m.backward(p.tokens.cuda(), p.h, dout, dh, dw_k=g["dw_k"], dw_v=g["dw_v"],
               dnorm_q=g["dnorm_q"], dnorm_k=g["dnorm_k"], dtables=g["dtables"], idx=idx,
               t_begin=sh.t_begin)
    torch.cuda.synchronize()
    assert m.check_errors() == 0
    return dh, g


def oracle_backward(p: Problem, rows, dout):
    sh = p.shape
    mini, zz = p.table_rows(rows)
    e = oracle.gather(mini, zz)
    rs = torch.from_numpy(rows).to(p.h.device)
    h = to_oracle(p.h[rs])
    g = dout[rs].double().cpu().numpy()
    b = oracle.backward(e, to_oracle(p.w_k_cpu), to_oracle(p.w_v_cpu), p.nq_cpu.numpy(),
                        p.nk_cpu.numpy(), h, g, 1e-6, round_dkv=sh.dtype == "bf16")
    b["dtables"] = oracle.table_grad(b["de"], p.z[rows], [int(x) for x in p.primes], sh.d_head)
    return b


def close(got, ref, dtype, what):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if dtype == "f32":
        err = np.abs(got - ref).max() if ref.size else 0.0
        assert err <= F32_TOL * max(1.0, np.abs(ref).max()), (what, err)
    else:
        err = rel_l2(got, ref)
        assert err <= BF16_REL, (what, err)


def check_all(p: Problem, dh, g, dout, rows=None, full=True):
    sh = p.shape
    rows = np.arange(sh.rows_out) if rows is None else rows
    b = oracle_backward(p, rows, dout)
    rs = torch.from_numpy(rows).cuda()
    if sh.dtype == "bf16":
        dh_ref = torch.from_numpy(b["dh"]).float().bfloat16().double().numpy()
        got = dh[rs].double().cpu().numpy()
        close(got, dh_ref, "bf16", "dh")
        assert np.mean(got == dh_ref) > 0.98
    else:
        close(dh[rs].cpu().numpy(), b["dh"], "f32", "dh")
    if not full:
        return
    for name in ("dw_k", "dw_v", "dnorm_q", "dnorm_k"):
        close(g[name].cpu().numpy(), b[name], sh.dtype, name)
    if g["dtables"] is not None:
        touched = 0
        for s, t in enumerate(g["dtables"]):
            zr = np.unique(p.z[rows, s])
            got = t.cpu().numpy()
            close(got[zr], b["dtables"][s][zr], sh.dtype, "dtable %d" % s)
            untouched = np.ones(got.shape[0], bool)
            untouched[zr] = False
            assert (got[untouched] == 0).all()
            touched += len(zr)
        assert touched > 0


def test_tiny_f32_all_gradients():
    p = Problem(synth.SHAPES["tiny_f32"])
    m = p.engram()
    dout = synth.make_grad_out(p.shape, p.seeds, device="cuda")
    dh, g = run_backward(p, m, dout)
    check_all(p, dh, g, dout)


@pytest.mark.parametrize("kw", [dict(), dict(d_hidden=256, branches=2),
                                dict(B=6, T=3, t_begin=2, branches=4)])
def test_bf16_reduced_all_gradients(kw):
    p = Problem(REDUCED.replace(**kw))
    m = p.engram()
    dout = synth.make_grad_out(p.shape, p.seeds, device="cuda")
    dh, g = run_backward(p, m, dout)
    check_all(p, dh, g, dout)


def test_accumulation_and_given_indices():
    p = Problem(REDUCED)
    m = p.engram()
    dout = synth.make_grad_out(p.shape, p.seeds, device="cuda")
    dh, g = run_backward(p, m, dout)
    first = {k: v.clone() for k, v in g.items() if k != "dtables"}
    tab = [t.clone() for t in g["dtables"]]
    idx = torch.empty((p.shape.rows_out, p.shape.num_tables), dtype=torch.int64, device="cuda")
    m.hash(p.tokens.cuda(), idx)
    dh2, g = run_backward(p, m, dout, idx=idx, grads=g)   # accumulates onto the first call
    assert torch.equal(dh2, dh)
    for k, v in first.items():
        assert rel_l2(g[k].double(), 2 * v.double()) < 1e-6, k
    for t, t0 in zip(g["dtables"], tab):
        assert rel_l2(t.double(), 2 * t0.double()) < 1e-6
    # without the optional outputs: dh only
    dh3, _ = run_backward(p, m, dout, grads=dict(dw_k=None, dw_v=None, dnorm_q=None,
                                                 dnorm_k=None, dtables=None))
    assert torch.equal(dh3, dh)


def test_prefill_full_size_sampled():
    # the benchmarked workload: dh on sampled rows against the oracle; the
    # weight gradients by homogeneity (every gradient is linear in dout)
    p = Problem(synth.SHAPES["prefill_bf16"])
    m = p.engram()
    dout = synth.make_grad_out(p.shape, p.seeds, device="cuda")
    dh, g = run_backward(p, m, dout, tables=False)
    check_all(p, dh, g, dout, rows=p.sample_rows(48), full=False)
    dh2, g2 = run_backward(p, m, 2 * dout, tables=False)
    for k in ("dw_k", "dw_v", "dnorm_q", "dnorm_k"):
        assert rel_l2(g2[k].double(), 2 * g[k].double()) < 1e-6, k
        assert torch.isfinite(g[k]).all() and g[k].abs().max() > 0


def test_prefill_full_size_sampled_rows_every_gradient():
    """The benchmarked workload and launch configuration (32 768 rows) with
    dL/dout zero outside a sample of rows: a row whose dout is zero has zero
    dk and dv (dv sums alpha dout over the branches, and d alpha = dout . v),
    so the weight, RMSNorm-weight and table gradients of the whole call equal
    the oracle's backward over the sampled rows alone, and dh is zero on every
    other row."""
    p = Problem(synth.SHAPES["prefill_bf16"])
    m = p.engram()
    rows = p.sample_rows(40, seed=5)
    mask = torch.zeros((p.shape.rows_out, 1, 1), device="cuda", dtype=torch.bfloat16)
    mask[torch.from_numpy(rows).cuda()] = 1
    dout = synth.make_grad_out(p.shape, p.seeds, device="cuda") * mask
    dh, g = run_backward(p, m, dout)
    check_all(p, dh, g, dout, rows=rows)
    others = torch.ones(p.shape.rows_out, dtype=torch.bool, device="cuda")
    others[torch.from_numpy(rows).cuda()] = False
    assert (dh[others] == 0).all()


def test_unsupported_modes():
    from hashed_gram_embedding_compress_b200 import engram as eg
    p = Problem(REDUCED.replace(T=40))
    dout = synth.make_grad_out(p.shape, p.seeds, device="cuda")
    m = p.engram()
    m.set_fp8(True)
    with pytest.raises(eg.EngramError) as ei:
        run_backward(p, m, dout)
    assert ei.value.code == eg.ENGRAM_ERR_UNSUPPORTED
    m = p.engram()
    cw, nw = p.conv_weights(4)
    m.set_short_conv(cw.cuda(), nw.cuda(), 4, 3)
    with pytest.raises(eg.EngramError) as ei:
        run_backward(p, m, dout)
    assert ei.value.code == eg.ENGRAM_ERR_UNSUPPORTED
