"""Host-side logic that needs no GPU: the projection-kernel choice of the
library (compiled from its header as plain C++) and the benchmark's
algorithmic work per step.
"""
import itertools
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "hashed_gram_embedding_compress_b200", "csrc")

_PROBE = r"""
#include "engram_internal.cuh"
#include <cstdio>
int main() {
  long long R;
  int phase, M, d, sms, flags, conv, wide;
  while (scanf("%d %lld %d %d %d %d %d %d", &phase, &R, &M, &d, &sms, &flags, &conv, &wide) == 8) {
    const engram::ProjChoice c = wide ? engram::wide_proj(phase, R, M, d, sms)
                                      : engram::choose_proj(phase, R, M, d, sms, flags, conv != 0);
    printf("%d %d %d %d\n", (int)c.kind, c.bn, c.grid, c.key_tile);
  }
  return 0;
}
"""
WIDE, PAIR, SINGLE = 0, 1, 2


@pytest.fixture(scope="module")
def choose(tmp_path_factory):
    d = tmp_path_factory.mktemp("choose")
    src, exe = d / "probe.cpp", d / "probe"
    src.write_text(_PROBE)
    subprocess.check_call(["g++", "-std=c++17", "-I", "/usr/local/cuda/include", "-I", CSRC,
                           str(src), "-o", str(exe)])

    def run(cases):
        inp = "".join("%d %d %d %d %d %d %d %d\n" % c for c in cases)
        out = subprocess.run([str(exe)], input=inp, capture_output=True, text=True, check=True)
        return [tuple(int(x) for x in line.split()) for line in out.stdout.splitlines()]
    return run


def test_prefill_uses_the_512x256_pair_tiles(choose):
    (k0, bn0, g0, kt0), (k1, _, g1, _) = choose([(0, 32768, 1, 2560, 148, 0, 0, 0),
                                                (1, 32768, 1, 2560, 148, 0, 0, 0)])
    assert (k0, bn0, g0, kt0) == (WIDE, 128, 148, 256) and (k1, g1) == (WIDE, 148)


def test_choice_invariants_over_shapes(choose):
    cases = [(ph, R, M, d, sms, fl, cv, 0)
             for ph, R, M, d, sms, fl, cv in itertools.product(
                 (0, 1), (1, 4, 256, 2048, 3000, 32768), (1, 2, 4), (128, 256, 512, 640, 2560, 4096),
                 (148, 132), (0, 1), (0, 1))]
    for c, (kind, bn, grid, kt) in zip(cases, choose(cases)):
        ph, R, M, d, sms, fl, cv, _ = c
        n_total = M * d if ph == 0 else d
        assert d % kt == 0, c                        # key tiles never straddle branches
        assert n_total % bn == 0 and 1 <= grid <= sms, c
        if fl:                                       # no CTA pairs: single-CTA tiles only
            assert kind == SINGLE, c
        if kind != SINGLE:
            assert grid % 2 == 0, c                  # whole CTA pairs
        if kind == WIDE:
            assert d % 256 == 0 and kt == 256, c
        if kind == PAIR:
            assert kt == 128 and not (ph == 1 and cv), c   # no pair kernel for the conv's values


def test_wide_choice_for_fp8(choose):
    cases = [(ph, R, M, d, 148, 0, 0, 1) for ph in (0, 1) for R in (1, 6, 513, 32768)
             for M in (1, 4) for d in (256, 2560)]
    for c, (kind, bn, grid, kt) in zip(cases, choose(cases)):
        ph, R, M, d = c[:4]
        tiles = -(-R // 512) * ((M * d if ph == 0 else d) // 256)
        assert (kind, bn, kt) == (WIDE, 128, 256) and grid == 2 * min(tiles, 74), c


def test_bench_algorithmic_work():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from hashed_gram_embedding_compress_b200 import synth
    sh = synth.SHAPES["prefill_bf16"]
    R, S = 32768, 16
    a = bench.algorithmic(sh)
    # tokens + S table rows of 160 bytes read and written per row
    assert a["gather_bytes"] == R * S * 160 * 2 + 8 * 4096 * 4 == 167903232
    assert a["gemm_flops"] == 2.0 * R * 1280 * (2560 + 2560)
    # FP8: codes (1 byte per element) and a 4-byte scale per row written instead of bf16 e
    assert bench.algorithmic(sh, fp8=True)["gather_bytes"] == R * S * 160 + R * 1284 + 8 * 4096 * 4
    # the step's unavoidable bytes: tokens, each addressed row once, h in, out, W once
    assert a["step_bytes"] == 8 * 4096 * 4 + R * S * 160 + 2 * R * 2560 * 2 + 2 * 2560 * 1280 * 2
    r = bench.step_roofline(a, 0.5, 6500.0, 1600.0)
    t_mma = a["gemm_flops"] / 1.6e15 * 1e3
    assert r["bound"] == "tensor" and abs(r["time_ms"] - t_mma) < 1e-12
    assert abs(r["frac"] - t_mma / 0.5) < 1e-12


def test_reference_arm_runs_the_oracle_without_the_library():
    """bench.py --impl reference times the oracle alone: the library's shared
    object is never loaded in its process."""
    import subprocess
    import sys
    code = (
        "import sys, types; sys.path.insert(0, %r); import bench\n"
        "a = types.SimpleNamespace(workload='tiny_f32', rows_target=None, short_conv=False,\n"
        "    fp8=False, backward=False, steps=1, warmup=0, cpu_seconds=0.2)\n"
        "r = bench.run_reference(a, 0, 1)\n"
        "assert r['impl'] == 'reference' and r['value'] > 0 and r['ms_per_step'] > 0\n"
        "maps = open('/proc/self/maps').read()\n"
        "assert 'libengram' not in maps and '_engram_oracle' in maps\n"
        "print('ok')\n" % ROOT)
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                         timeout=300, env=dict(os.environ, CUDA_VISIBLE_DEVICES=""))
    assert out.returncode == 0 and "ok" in out.stdout, out.stderr[-2000:]


def _cpu_problem():
    import oracle
    from hashed_gram_embedding_compress_b200 import synth
    sh = synth.SHAPES["tiny_f32"]
    seeds = synth.stream_seeds(sh)
    primes = oracle.table_primes(sh.rows_target, sh.num_tables)
    w_k, w_v, nq, nk = synth.make_weights(sh, seeds)
    P = dict(sh=sh, tokens=synth.make_tokens(sh, seeds), comp_map=synth.make_comp_map(sh, seeds),
             hash_seed=synth.make_hash_seed(seeds), w_k=w_k, w_v=w_v, nq=nq, nk=nk,
             tables=synth.make_tables([int(p) for p in primes], sh.d_head, sh.dtype, seeds,
                                      device="cpu"),
             h=synth.make_hidden(sh, seeds), conv=None)
    return P, synth.make_grad_out(sh, seeds)


def test_cpu_baselines_run_the_oracle_on_a_bounded_sample():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    P, dout = _cpu_problem()
    f = bench.cpu_baseline(P, 0.3)
    b = bench.cpu_baseline_backward(P, dout, 0.3)
    for r in (f, b):
        assert r["kind"] == "oracle" and r["cores"] == 1 and r["value"] > 0
    assert "backward" in b["sample"] and "backward" not in f["sample"]
