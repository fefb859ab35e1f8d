"""engram_project_gate_noalloc: the allocation-free projection + gate.

For callers that cannot let the library allocate device memory (work issued
during CUDA graph capture, hosts that own every device allocation).  Its
output must match engram_forward's within the tolerance of the parity tests,
and the oracle's on sampled rows, on two calls in a row.  The second call
gets other hidden states than the first, so a value phase that read partial
sums left in the library's fixed scratch array by the first call would give
the wrong gate.
"""
import numpy as np
import pytest
import torch

import oracle
from engram_cases import Problem, out_close, rel_l2, to_oracle
from hashed_gram_embedding_compress_b200 import synth

pytestmark = pytest.mark.gpu

BF16_REL = 1e-3
F32_ABS = 1e-5


def _inputs(p: Problem, m):
    sh = p.shape
    idx = torch.empty((sh.rows_out, sh.num_tables), dtype=torch.int64, device="cuda")
    e = torch.empty((sh.rows_out, sh.d_mem), dtype=synth.torch_dtype(sh.dtype), device="cuda")
    m.hash(p.tokens.cuda(), idx, t_begin=sh.t_begin)
    m.gather(idx, e)
    return e


def _close(x, ref, f32: bool) -> bool:
    if f32:
        return float((x.double() - ref.double()).abs().max()) <= F32_ABS
    return rel_l2(x.double(), ref.double()) <= BF16_REL


def _oracle_rows(p: Problem, h: torch.Tensor, rows: np.ndarray):
    """alpha and out of the oracle at `rows`, for hidden states h."""
    mini, zz = p.table_rows(rows)
    e = oracle.gather(mini, zz)
    hr = to_oracle(h[torch.from_numpy(rows).to(h.device)])
    alpha, _, out = oracle.project_gate(e, to_oracle(p.w_k_cpu), to_oracle(p.w_v_cpu),
                                        p.nq_cpu.numpy(), p.nk_cpu.numpy(), hr, 1e-6)
    return alpha, out


@pytest.mark.parametrize("shape", [
    # CTA-pair tiles: 6000 rows, d = 2560, one branch
    synth.SHAPES["prefill_bf16"].replace(B=1, T=6000, rows_target=4099),
    # single-CTA tiles: 256 decode rows, four branches
    synth.SHAPES["decode_mb"].replace(rows_target=4099),
    # fp32 SIMT path
    synth.SHAPES["tiny_f32"],
])
def test_noalloc_matches_forward_and_oracle_on_two_calls(shape):
    p = Problem(shape)
    m = p.engram()
    sh = p.shape
    R, M = sh.rows_out, sh.branches
    f32 = sh.dtype == "f32"
    e = _inputs(p, m)
    # the second call's hidden states: another seeded draw of the same shape
    h2 = synth.make_hidden(sh, synth.stream_seeds(sh, extra=7), device="cuda")
    rows = p.sample_rows(48, seed=3)
    for h in (p.h, h2):
        ref = torch.empty_like(h)
        a_ref = torch.empty((R, M), device="cuda")
        m.forward(p.tokens.cuda(), h, ref, t_begin=sh.t_begin, alpha=a_ref)
        out = torch.full_like(h, float("nan"))
        alpha = torch.full((R, M), -1.0, device="cuda")
        m.project_gate_noalloc(e, h, out, alpha=alpha)
        torch.cuda.synchronize()
        assert m.check_errors() == 0
        assert not torch.isnan(out.float()).any()
        assert _close(out, ref, f32)
        assert _close(alpha, a_ref, f32)
        a_o, o_o = _oracle_rows(p, h, rows)
        a_g = alpha[torch.from_numpy(rows).cuda()].double().cpu().numpy()
        o_g = to_oracle(out[torch.from_numpy(rows).cuda()])
        if f32:
            assert float(np.abs(a_g - a_o).max()) <= F32_ABS
            assert out_close(o_g, o_o, "f32") <= F32_ABS
        else:
            assert rel_l2(a_g, a_o) <= BF16_REL
            assert out_close(o_g, o_o, "bf16") <= BF16_REL


def test_noalloc_rejects_rows_beyond_its_scratch():
    from hashed_gram_embedding_compress_b200 import engram as eg
    sh = synth.SHAPES["prefill_bf16"].replace(B=1, T=64, rows_target=1031)
    p = Problem(sh)
    m = p.engram()
    limit = (4 << 20) // (16 * sh.branches * sh.d_hidden // 64)
    e = torch.zeros((limit + 1, sh.d_mem), dtype=torch.bfloat16, device="cuda")
    h = torch.zeros((limit + 1, sh.branches, sh.d_hidden), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(eg.EngramError) as ei:
        m.project_gate_noalloc(e, h, h)
    assert ei.value.code == eg.ENGRAM_ERR_INVALID and str(limit) in str(ei.value)
    # at the limit it runs
    m.project_gate_noalloc(e[:limit], h[:limit], h[:limit])
    torch.cuda.synchronize()
    assert m.check_errors() == 0


def test_noalloc_binding_checks_shapes_before_the_call():
    from hashed_gram_embedding_compress_b200 import engram as eg
    sh = synth.SHAPES["prefill_bf16"].replace(B=1, T=64, rows_target=1031)
    p = Problem(sh)
    m = p.engram()
    e = torch.zeros((64, sh.d_mem), dtype=torch.bfloat16, device="cuda")
    h = torch.zeros((64, sh.branches, sh.d_hidden), dtype=torch.bfloat16, device="cuda")
    for bad in (dict(h=h[:32]), dict(out=h[:32]), dict(h=h.float()),
                dict(alpha=torch.zeros((64, sh.branches + 1), device="cuda"))):
        args = dict(e=e, h=h, out=h) | bad
        with pytest.raises(eg.EngramError) as ei:
            m.project_gate_noalloc(args["e"], args["h"], args["out"], alpha=args.get("alpha"))
        assert ei.value.code == eg.ENGRAM_ERR_INVALID
