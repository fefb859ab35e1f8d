"""The C-ABI library: loads, exports every declared symbol, validates configs.

No compute calls: these run without a GPU.  A config that passes validation
fails only at its first CUDA call (ENGRAM_ERR_CUDA) on a machine with no GPU.
"""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def eg():
    from hashed_gram_embedding_compress_b200 import build
    build.build()
    from hashed_gram_embedding_compress_b200 import engram
    return engram


def declared_symbols():
    hdr = open(os.path.join(ROOT, "include", "engram.h")).read()
    return set(re.findall(r"ENGRAM_API[^;(]*?\b(engram_\w+)\s*\(", hdr))


def test_header_and_binding_agree(eg):
    names = declared_symbols()
    assert names == set(eg.EXPORTS) and len(names) == 31


def test_library_exports_every_declared_symbol(eg):
    L = ctypes.CDLL(eg.LIB_PATH)
    for n in declared_symbols():
        assert hasattr(L, n), n
    out = os.popen("nm -D --defined-only %s" % eg.LIB_PATH).read()
    exported = set(re.findall(r"\bT (engram_\w+)", out))
    assert exported == declared_symbols()


def test_config_layout(eg):
    assert eg.lib.engram_config_size() == ctypes.sizeof(eg.engram_config) == 600


def _cfg(eg, **kw):
    args = dict(vocab=100, cvocab=80, comp_map=torch.arange(100) % 80, orders=(2, 3), heads=2,
                d_head=32, d_hidden=128, branches=1, dtype="f32", table_rows_target=101)
    args.update(kw)
    return eg.make_config(**args)


@pytest.mark.parametrize("kw,msg", [
    (dict(cvocab=101), "cvocab"),
    (dict(vocab=0, cvocab=0, comp_map=torch.zeros(1)), "cvocab"),
    (dict(orders=(3, 2)), "ascending"),
    (dict(orders=(2, 5)), "orders"),
    (dict(heads=0), "heads"),
    (dict(heads=33), "heads"),
    (dict(d_head=6), "d_head"),
    (dict(d_head=4, dtype="bf16"), "d_head"),
    (dict(d_hidden=96), "d_hidden"),
    (dict(branches=5), "branches"),
    (dict(branches=0), "branches"),
    (dict(eps=float("nan")), "eps"),
    (dict(table_rows_target=1), "table_rows_target"),
    (dict(primes=[101, 0, 103, 107]), "all table sizes"),
    (dict(primes=[101, 1, 103, 107]), "table sizes"),
    (dict(comp_map=torch.arange(100)), "comp_map"),
    (dict(pad_id=-2), "pad_id"),
    (dict(flags=4), "unknown flags"),
])
def test_invalid_configs_rejected_before_any_cuda_call(eg, kw, msg):
    cfg = _cfg(eg, **kw)
    with pytest.raises(eg.EngramError) as ei:
        eg.Engram(cfg)
    assert ei.value.code == eg.ENGRAM_ERR_INVALID
    assert msg in str(ei.value)


def test_null_arguments(eg):
    h = ctypes.c_void_p()
    assert eg.lib.engram_create(None, ctypes.byref(h)) == eg.ENGRAM_ERR_INVALID
    for fn, args in (("engram_reserve", (None, 1)),
                     ("engram_hash", (None, None, 1, 1, 0, None, None)),
                     ("engram_forward", (None, None, None, 1, 1, 0) + (None,) * 5),
                     ("engram_check_errors", (None, None)),
                     ("engram_set_params", (None,) * 6),
                     ("engram_gather", (None, None, 1, None, None)),
                     ("engram_prefetch", (None, None, 1, 1, 0, None, None)),
                     ("engram_profile_next_forward", (None, None, 5)),
                     ("engram_project_gate_noalloc", (None, None, 1, None, None, None, None)),
                     ("engram_selftest_timeout", (None, None)),
                     ("engram_set_short_conv", (None, None, None, 4, 3, None)),
                     ("engram_build_hot_cache", (None, None, 1, 1, 0, 1, None)),
                     ("engram_prefetch_hot_hits", (None, None)),
                     ("engram_set_fp8", (None, 1, None)),
                     ("engram_quantize_e4m3", (None, None, 1, 16, None, None, None)),
                     ("engram_backward", (None, None, None, 1, 1, 0) + (None,) * 9),
                     ("engram_profile_next_backward", (None, None, 6))):
        assert getattr(eg.lib, fn)(*args) == eg.ENGRAM_ERR_INVALID, fn
    assert eg.lib.engram_kernel_launches(None) == -1
    eg.lib.engram_destroy(None)


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_valid_config_without_gpu_fails_with_cuda_error(eg):
    with pytest.raises(eg.EngramError) as ei:
        eg.Engram(_cfg(eg))
    assert ei.value.code in (eg.ENGRAM_ERR_CUDA, eg.ENGRAM_ERR_OOM)
