"""engram_project_gate_noalloc: the allocation-free projection + gate.

For callers that cannot let the library allocate device memory (work issued
during CUDA graph capture, hosts that own every device allocation).  Its
output must match engram_forward's within the tolerance of the parity tests,
on two calls in a row (the second call reuses the library's fixed scratch
array, which still holds the first call's partial sums).
"""
import pytest
import torch

from engram_cases import Problem, rel_l2
from hashed_gram_embedding_compress_b200 import synth

pytestmark = pytest.mark.gpu

BF16_REL = 1e-3


def _inputs(p: Problem, m):
    sh = p.shape
    idx = torch.empty((sh.rows_out, sh.num_tables), dtype=torch.int64, device="cuda")
    e = torch.empty((sh.rows_out, sh.d_mem), dtype=synth.torch_dtype(sh.dtype), device="cuda")
    m.hash(p.tokens.cuda(), idx, t_begin=sh.t_begin)
    m.gather(idx, e)
    return e


@pytest.mark.parametrize("shape", [
    # CTA-pair tiles: 6000 rows, d = 2560, one branch
    synth.SHAPES["prefill_bf16"].replace(B=1, T=6000, rows_target=4099),
    # single-CTA tiles: 256 decode rows, four branches
    synth.SHAPES["decode_mb"].replace(rows_target=4099),
])
def test_noalloc_matches_forward_on_two_calls(shape):
    p = Problem(shape)
    m = p.engram()
    sh = p.shape
    R, M = sh.rows_out, sh.branches
    ref = torch.empty_like(p.h)
    a_ref = torch.empty((R, M), device="cuda")
    m.forward(p.tokens.cuda(), p.h, ref, t_begin=sh.t_begin, alpha=a_ref)
    e = _inputs(p, m)
    for _ in range(2):
        out = torch.full_like(p.h, float("nan"))
        alpha = torch.full((R, M), -1.0, device="cuda")
        m.project_gate_noalloc(e, p.h, out, alpha=alpha)
        torch.cuda.synchronize()
        assert m.check_errors() == 0
        assert rel_l2(out.double(), ref.double()) <= BF16_REL
        assert rel_l2(alpha.double(), a_ref.double()) <= BF16_REL
        assert not torch.isnan(out.float()).any()


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
