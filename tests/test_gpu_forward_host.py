"""The forward from host buffers (engram_forward_host): the library stages
tokens and h on the device, runs the same forward in place, and copies out and
alpha back.  Its results must equal the device-buffer forward bit for bit,
call after call, while the two stagings alternate and one call's copies in
overlap the previous call's copies out."""
import pytest
import torch

from engram_cases import Problem, out_close, rel_l2, to_oracle
from hashed_gram_embedding_compress_b200 import synth

pytestmark = pytest.mark.gpu

SHAPE = synth.SHAPES["prefill_bf16"].replace(B=2, T=300, rows_target=4099, d_hidden=512)


def _device_forward(m, tok, h):
    out = torch.empty_like(h)
    alpha = torch.empty((h.shape[0], h.shape[1]), device="cuda")
    m.forward(tok, h, out, alpha=alpha)
    return out, alpha


def test_host_buffers_equal_device_forward_over_several_calls():
    p = Problem(SHAPE)
    m = p.engram()
    tok_h = p.tokens.pin_memory()
    tok_d = p.tokens.cuda()
    # three calls with different h, issued back to back before any check
    hs = [p.h.cpu()]
    for k in range(2):
        g = torch.Generator().manual_seed(1000 + k)
        hs.append((torch.randn(p.h.shape, generator=g) * 0.5).to(p.h.dtype))
    hs_pinned = [x.pin_memory() for x in hs]
    outs = [torch.empty_like(x).pin_memory() for x in hs]
    alphas = [torch.empty((x.shape[0], x.shape[1]), dtype=torch.float32).pin_memory() for x in hs]
    for x, o, a in zip(hs_pinned, outs, alphas):
        m.forward_host(tok_h, x, o, alpha=a)
    torch.cuda.synchronize()
    assert m.check_errors() == 0
    for x, o, a in zip(hs, outs, alphas):
        ref, a_ref = _device_forward(m, tok_d, x.cuda())
        torch.cuda.synchronize()
        assert torch.equal(o, ref.cpu()) and torch.equal(a, a_ref.cpu())
    # the first call against the oracle on sampled rows
    rows = p.sample_rows(16)
    _, a_o, _, o_o = p.oracle_forward(rows)
    rs = torch.from_numpy(rows)
    assert rel_l2(alphas[0][rs].double(), a_o) <= 1e-3
    assert out_close(to_oracle(outs[0][rs]), o_o, "bf16") <= 1e-3


def test_host_buffers_in_place_pageable_and_decode_rows():
    p = Problem(SHAPE)
    m = p.engram()
    tok = p.tokens.clone()
    x = p.h.cpu().clone()  # pageable, updated in place (out is h)
    ref, _ = _device_forward(m, p.tokens.cuda(), p.h)
    m.forward_host(tok, x, x)
    torch.cuda.synchronize()
    assert torch.equal(x, ref.cpu())
    # the newest position only (t_begin = T - 1)
    T = tok.shape[1]
    xh = p.h.cpu()[: tok.shape[0]].clone()
    out = torch.empty_like(xh)
    m.forward_host(tok, xh, out, t_begin=T - 1)
    ref2 = torch.empty_like(xh.cuda())
    m.forward(p.tokens.cuda(), xh.cuda(), ref2, t_begin=T - 1)
    torch.cuda.synchronize()
    assert m.check_errors() == 0 and torch.equal(out, ref2.cpu())


def test_host_buffers_reject_device_tensors_and_bad_shapes():
    from hashed_gram_embedding_compress_b200 import engram as eg
    p = Problem(SHAPE)
    m = p.engram()
    with pytest.raises(eg.EngramError) as ei:
        m.forward_host(p.tokens, p.h, torch.empty_like(p.h).cpu())  # h on the device
    assert ei.value.code == eg.ENGRAM_ERR_INVALID
    with pytest.raises(eg.EngramError) as ei:
        m.forward_host(p.tokens, p.h.cpu()[:-1], torch.empty_like(p.h).cpu()[:-1])
    assert ei.value.code == eg.ENGRAM_ERR_INVALID
    with pytest.raises(eg.EngramError) as ei:
        m.forward_host(p.tokens, p.h.cpu().float(), torch.empty_like(p.h).cpu().float())
    assert ei.value.code == eg.ENGRAM_ERR_INVALID


def test_backward_host_buffers_equal_device_backward():
    """engram_backward_host: h and dout in, dh out through host buffers, two
    calls back to back; dh equal to the device-buffer backward bit for bit and
    the weight gradients accumulated once per call."""
    p = Problem(SHAPE)
    sh = p.shape
    M, d, dm = sh.branches, sh.d_hidden, sh.d_mem
    m = p.engram()
    dout = synth.make_grad_out(sh, p.seeds, device="cpu")
    tok_h, h_h, g_h = p.tokens.pin_memory(), p.h.cpu().pin_memory(), dout.pin_memory()
    dh1, dh2 = torch.empty_like(h_h).pin_memory(), torch.empty_like(h_h).pin_memory()
    dw_v = torch.zeros((d, dm), device="cuda")
    m.backward_host(tok_h, h_h, g_h, dh1, dw_v=dw_v)
    m.backward_host(tok_h, h_h, g_h, dh2, dw_v=dw_v)
    torch.cuda.synchronize()
    assert m.check_errors() == 0
    ref = torch.empty_like(p.h)
    dw_ref = torch.zeros((d, dm), device="cuda")
    m.backward(p.tokens.cuda(), p.h, dout.cuda(), ref, dw_v=dw_ref)
    torch.cuda.synchronize()
    assert torch.equal(dh1, ref.cpu()) and torch.equal(dh2, ref.cpu())
    # two accumulations of the same gradient (the contraction's order may vary in the last bits)
    assert rel_l2((dw_v / 2).double().cpu(), dw_ref.double().cpu()) < 1e-6
