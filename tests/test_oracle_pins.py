"""Pins of the CPU oracle against what the pages and mathematics fix.

Each test checks the oracle against something other than itself: a published
test sequence, hand-derived worked examples, closed forms of Eq. (4), an
independent library (sympy, numpy indexing, torch fp64 matmul), brute-force
enumeration and the uniform-hash expectation.
"""
import json
import math
import os

import numpy as np
import pytest
import sympy
import torch

import oracle


def _sig(x):
    return 1.0 / (1.0 + math.exp(-x))


# --------------------------------------------------------------- SplitMix64

def test_splitmix64_published_sequence(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "splitmix64_seed1234567.json")))
    assert oracle.splitmix64_stream(g["seed"], 5) == [int(v) for v in g["outputs"]]


def test_multipliers_are_the_stream_forced_odd():
    seed, S, J = 1234567, 3, 3
    m = oracle.hash_multipliers(seed, S, J)
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                    "splitmix64_seed1234567.json")))
    first = [int(v) | 1 for v in g["outputs"]]
    assert [int(x) for x in m.reshape(-1)[:5]] == first
    assert all(int(x) & 1 for x in m.reshape(-1))
    assert len({int(x) for x in m.reshape(-1)}) == S * J


# ------------------------------------------------------------------- primes

@pytest.mark.parametrize("target,S", [(10007, 8), (1 << 20, 16), (1 << 24, 16), (2, 5), (90, 4)])
def test_table_primes_match_sympy(target, S):
    p = oracle.table_primes(target, S)
    want, n = [], target - 1
    for _ in range(S):
        n = sympy.nextprime(n)
        want.append(n)
    assert [int(x) for x in p] == want


def test_known_primes_above_powers_of_two():
    # smallest primes above 2^20 and 2^24 are 2^20 + 7 and 2^24 + 43
    assert int(oracle.table_primes(1 << 20, 1)[0]) == (1 << 20) + 7
    assert int(oracle.table_primes(1 << 24, 1)[0]) == (1 << 24) + 43
    assert oracle.is_prime(10007) and not oracle.is_prime(10005) and not oracle.is_prime(1)


# -------------------------------------------------------------- compression

def test_compress_lookup_and_range_error():
    m = np.array([2, 0, 1, 0], dtype=np.int32)
    x = np.array([[0, 1, 2, 3, 3]], dtype=np.int32)
    assert oracle.compress(x, m).tolist() == [[2, 0, 1, 0, 0]]
    with pytest.raises(ValueError):
        oracle.compress(np.array([[4]], dtype=np.int32), m)
    with pytest.raises(ValueError):
        oracle.compress(np.array([[-1]], dtype=np.int32), m)


# ------------------------------------------------------------------ hashing

def test_hash_worked_examples(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "hash_worked_examples.json")))
    for case in g["cases"]:
        mult = np.array([[int(v) for v in row] for row in case["mult"]], dtype=np.uint64)
        z = oracle.hash_indices(np.array(case["c"], dtype=np.int32), case["pad"], case["orders"],
                                case["heads"], mult, np.array(case["primes"], dtype=np.int64))
        assert z.tolist() == case["z"], case["name"]


def test_hash_t_begin_emits_suffix_rows_only():
    rng = np.random.default_rng(0)
    c = rng.integers(0, 50, size=(3, 7)).astype(np.int32)
    mult = oracle.hash_multipliers(99, 4, 3)
    primes = oracle.table_primes(211, 4)
    full = oracle.hash_indices(c, 50, (2, 3), 2, mult, primes).reshape(3, 7, 4)
    tail = oracle.hash_indices(c, 50, (2, 3), 2, mult, primes, t_begin=5).reshape(3, 2, 4)
    assert np.array_equal(full[:, 5:], tail)


def test_hash_invariants_identical_ngrams_same_rows():
    rng = np.random.default_rng(1)
    B, T, V = 4, 200, 12
    c = rng.integers(0, V, size=(B, T)).astype(np.int32)
    mult = oracle.hash_multipliers(7, 6, 3)
    primes = oracle.table_primes(1009, 6)
    z = oracle.hash_indices(c, V, (2, 3), 3, mult, primes).reshape(B, T, 6)
    assert (z >= 0).all() and (z < primes[None, None, :]).all()
    padded = np.concatenate([np.full((B, 2), V, np.int32), c], axis=1)
    seen = {}
    for b in range(B):
        for t in range(T):
            g2 = tuple(padded[b, t + 1:t + 3])
            g3 = tuple(padded[b, t:t + 3])
            for key, val in (((2,) + g2, tuple(z[b, t, :3])), ((3,) + g3, tuple(z[b, t, 3:]))):
                assert seen.setdefault(key, val) == val
    # different heads of one order use different multipliers, so they disagree somewhere
    assert (z[:, :, 0] != z[:, :, 1]).any()


def _all_ngrams(V, n):
    grid = np.stack(np.meshgrid(*[np.arange(V)] * n, indexing="ij"), -1).reshape(-1, n)
    return grid.astype(np.int32)


@pytest.mark.parametrize("n,p", [(2, 101), (2, 1009), (3, 100003), (3, 1009)])
def test_hash_collisions_brute_force_and_uniform_expectation(n, p):
    V = 41  # 40 compressed ids and the pad id
    seqs = _all_ngrams(V, n)
    D = seqs.shape[0]
    mult = oracle.hash_multipliers(20261202, 1, 3)
    z = oracle.hash_indices(seqs, V - 1, (n,), 1, mult, np.array([p], np.int64),
                            t_begin=n - 1)[:, 0]
    # brute-force enumeration of colliding pairs
    pairs = 0
    for i in range(0, D, 4096):
        blk = z[i:i + 4096]
        pairs += int((blk[:, None] == z[None, :]).sum()) - blk.size
    pairs //= 2
    counts = np.bincount(z, minlength=p)
    assert pairs == int((counts * (counts - 1) // 2).sum())
    # uniform hashing: E[pairs] = C(D,2)/p, Var ~ E (1 - 1/p)
    exp_pairs = D * (D - 1) / 2 / p
    assert abs(pairs - exp_pairs) < 5 * math.sqrt(exp_pairs * (1 - 1 / p)) + 1
    occ = int((counts > 0).sum())
    exp_occ = p * (1 - (1 - 1 / p) ** D)
    assert abs(occ - exp_occ) < 5 * math.sqrt(max(exp_occ * (1 - exp_occ / p), 1.0)) + 2


# ------------------------------------------------------------------- gather

@pytest.mark.parametrize("dtype", [np.float32, np.uint16])
def test_gather_matches_numpy_indexing(dtype):
    rng = np.random.default_rng(2)
    S, d_h, rows = 5, 7, 33
    tabs = [rng.integers(0, 60000, size=(97 + s, d_h)).astype(dtype) for s in range(S)]
    z = np.stack([rng.integers(0, 97 + s, size=rows) for s in range(S)], 1)
    e = oracle.gather(tabs, z)
    want = np.concatenate([tabs[s][z[:, s]] for s in range(S)], axis=1)
    assert e.dtype == want.dtype and np.array_equal(e, want)
    with pytest.raises(IndexError):
        oracle.gather(tabs, np.full((1, S), 97 + S, dtype=np.int64))


# --------------------------------------------------------------- projection

def _bf16_bits(x: torch.Tensor) -> np.ndarray:
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_project_matches_torch_fp64():
    g = torch.Generator().manual_seed(3)
    e = torch.randn(9, 40, generator=g)
    w = torch.randn(13, 40, generator=g)
    y = oracle.project(e.numpy(), w.numpy())
    ref = (e.double() @ w.double().T).numpy()
    assert np.allclose(y, ref, rtol=1e-13, atol=1e-13)
    yb = oracle.project(_bf16_bits(e), _bf16_bits(w))
    refb = (e.bfloat16().double() @ w.bfloat16().double().T).numpy()
    assert np.allclose(yb, refb, rtol=1e-13, atol=1e-13)


# --------------------------------------------------------------------- gate

def test_gate_worked_examples(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "gate_worked_examples.json")))
    for case in g["cases"]:
        s = eval(case["s"], {"sqrt": math.sqrt})
        a = oracle.gate(np.array(case["h"], float), np.array(case["k"], float),
                        np.array(case["wq"], np.float32), np.array(case["wk"], np.float32),
                        case["eps"])
        assert abs(a - _sig(s)) < 1e-14, case["name"]


def test_gate_scale_invariance_and_range():
    rng = np.random.default_rng(4)
    d = 64
    h, k = rng.normal(size=d), rng.normal(size=d)
    wq = (1 + 0.1 * rng.normal(size=d)).astype(np.float32)
    wk = (1 + 0.1 * rng.normal(size=d)).astype(np.float32)
    a = oracle.gate(h, k, wq, wk, 0.0)
    assert 0.0 < a < 1.0
    assert abs(oracle.gate(5.0 * h, 0.25 * k, wq, wk, 0.0) - a) < 1e-14
    assert abs(oracle.gate(-h, k, wq, wk, 0.0) - (1 - a)) < 1e-14


# --------------------------------------------------------------- full gate

def _small_problem(M=2, d=16, dm=24, rows=5, seed=5, bf16=False):
    g = torch.Generator().manual_seed(seed)
    e = torch.randn(rows, dm, generator=g) * 0.5
    wk = torch.randn(M, d, dm, generator=g) / math.sqrt(dm)
    wv = torch.randn(d, dm, generator=g) / math.sqrt(dm)
    h = torch.randn(rows, M, d, generator=g)
    nq = 1 + 0.1 * torch.randn(M, d, generator=g)
    nk = 1 + 0.1 * torch.randn(M, d, generator=g)
    if bf16:
        cv = _bf16_bits
    else:
        cv = lambda t: t.float().numpy()
    return cv(e), cv(wk), cv(wv), nq.numpy(), nk.numpy(), cv(h), (e, wk, wv, h)


@pytest.mark.parametrize("bf16", [False, True])
def test_project_gate_against_torch_fp64(bf16):
    e, wk, wv, nq, nk, h, raw = _small_problem(bf16=bf16)
    alpha, delta, out = oracle.project_gate(e, wk, wv, nq, nk, h, 1e-6)
    conv = (lambda t: t.bfloat16().double()) if bf16 else (lambda t: t.double())
    E, WK, WV, H = [conv(t) for t in raw]
    k = torch.einsum("rj,mij->rmi", E, WK)
    v = E @ WV.T
    d = H.shape[-1]
    qn = H / torch.sqrt(H.pow(2).mean(-1, keepdim=True) + 1e-6) * torch.from_numpy(nq).double()
    kn = k / torch.sqrt(k.pow(2).mean(-1, keepdim=True) + 1e-6) * torch.from_numpy(nk).double()
    a_ref = torch.sigmoid((qn * kn).sum(-1) / math.sqrt(d))
    assert np.allclose(alpha, a_ref.numpy(), rtol=1e-12, atol=1e-12)
    d_ref = a_ref[..., None] * v[:, None, :]
    assert np.allclose(delta, d_ref.numpy(), rtol=1e-12, atol=1e-12)
    o_ref = H + d_ref
    if bf16:
        want = _bf16_bits(o_ref.float())
        assert np.array_equal(out, want)
    else:
        assert np.array_equal(out, o_ref.float().numpy())


def test_project_gate_zero_value_projection_keeps_h():
    e, wk, wv, nq, nk, h, _ = _small_problem()
    alpha, delta, out = oracle.project_gate(e, wk, np.zeros_like(wv), nq, nk, h, 1e-6)
    assert np.array_equal(out, h) and (delta == 0).all()
    assert ((alpha > 0) & (alpha < 1)).all()


def test_project_gate_shared_value_per_branch():
    # Eq. (6): branches share W_V; identical W_K and h in both branches give equal alpha
    e, wk, wv, nq, nk, h, _ = _small_problem(M=2)
    wk[1] = wk[0]
    h[:, 1] = h[:, 0]
    nq[1] = nq[0]
    nk[1] = nk[0]
    alpha, delta, _ = oracle.project_gate(e, wk, wv, nq, nk, h, 1e-6)
    assert np.array_equal(alpha[:, 0], alpha[:, 1])
    assert np.array_equal(delta[:, 0], delta[:, 1])


# ------------------------------------------------------------ ShortConv (Eq. 5)

def _conv_case(seed, n_pos=41, d=24, W=4):
    rng = np.random.default_rng(seed)
    vt = rng.normal(size=(n_pos, d)) * rng.uniform(0.1, 3.0, size=(n_pos, 1))
    cw = rng.normal(size=(d, W)).astype(np.float32)
    nw = (1 + 0.1 * rng.normal(size=d)).astype(np.float32)
    return vt, cw, nw


@pytest.mark.parametrize("dil,W", [(3, 4), (2, 4), (1, 3), (4, 2)])
def test_short_conv_matches_library_routines(dil, W):
    # RMSNorm, a causal dilated depthwise conv1d and SiLU from torch, in fp64:
    # torch's conv1d is a cross-correlation, so its kernel is the oracle's
    # taps reversed, and left padding of (W-1) dil makes it causal
    vt, cw, nw = _conv_case(dil * 10 + W, W=W)
    eps = 1e-6
    y = oracle.short_conv(vt, cw, nw, dil, eps)
    x = torch.from_numpy(vt)
    n = torch.nn.functional.rms_norm(x, (x.shape[1],), weight=torch.from_numpy(nw).double(), eps=eps)
    k = torch.from_numpy(cw).double().flip(1).unsqueeze(1)           # [d, 1, W]
    xin = torch.nn.functional.pad(n.T.unsqueeze(0), ((W - 1) * dil, 0))
    conv = torch.nn.functional.conv1d(xin, k, groups=x.shape[1], dilation=dil)[0].T
    ref = torch.nn.functional.silu(conv) + x
    assert np.abs(y - ref.numpy()).max() < 1e-12


def test_short_conv_zero_weights_is_identity():
    # the paper's zero initialisation: SiLU(0) = 0, so Y = V~ exactly
    vt, cw, nw = _conv_case(1)
    y = oracle.short_conv(vt, np.zeros_like(cw), nw, 3, 1e-6)
    assert np.array_equal(y, vt)


def test_short_conv_causal_dilated_support():
    # a change of V~ at position p moves Y exactly at p, p+dil, ..., p+(W-1)dil
    vt, cw, nw = _conv_case(2, n_pos=40)
    y0 = oracle.short_conv(vt, cw, nw, 3, 1e-6)
    for p in (0, 5, 33):
        v2 = vt.copy()
        v2[p] *= 1.7
        v2[p, 3] += 0.5
        y1 = oracle.short_conv(v2, cw, nw, 3, 1e-6)
        changed = set(np.nonzero(np.abs(y1 - y0).max(axis=1) > 0)[0].tolist())
        assert changed == {q for q in (p, p + 3, p + 6, p + 9) if q < 40}


def test_short_conv_at_equals_sequence_form():
    vt, cw, nw = _conv_case(3)
    y = oracle.short_conv(vt, cw, nw, 3, 1e-6)
    for t in (0, 2, 3, 8, 9, 40):
        taps = np.stack([vt[t - 3 * i] if t - 3 * i >= 0 else np.zeros(vt.shape[1]) for i in range(4)])
        have = np.array([t - 3 * i >= 0 for i in range(4)], dtype=np.int32)
        assert np.array_equal(oracle.short_conv_at(taps, have, cw, nw, 1e-6), y[t])


def test_add_round_matches_torch_rounding():
    rng = np.random.default_rng(4)
    hb = torch.randn(4096, dtype=torch.float64).to(torch.bfloat16)
    y = rng.normal(size=4096) * 0.01
    out = oracle.add_round(hb.view(torch.int16).numpy().view(np.uint16), y)
    ref = (hb.double() + torch.from_numpy(y)).float().to(torch.bfloat16)
    assert np.array_equal(out, ref.view(torch.int16).numpy().view(np.uint16))
    hf = rng.normal(size=100).astype(np.float32)
    assert np.array_equal(oracle.add_round(hf, y[:100]), (hf.astype(np.float64) + y[:100]).astype(np.float32))


# ------------------------------------------------- FP8 projection (section 2.4)

def _torch_e4m3(x32: np.ndarray) -> np.ndarray:
    """E4M3 codes from torch's own float -> float8_e4m3fn conversion."""
    return torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).to(
        torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_decode_matches_torch_on_every_code():
    codes = np.arange(256, dtype=np.uint8)
    v = oracle.e4m3_decode(codes)
    t = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(v), np.isnan(t)) and np.isnan(v).sum() == 2
    assert np.array_equal(v[~np.isnan(v)], t[~np.isnan(t)])
    # the format's fixed points: largest finite 448, smallest subnormal 2^-9, smallest normal 2^-6
    assert v[0x7E] == 448.0 and v[0x01] == 2.0 ** -9 and v[0x08] == 2.0 ** -6
    assert np.array_equal(v[0x80:0xFE], -v[0x00:0x7E])


def test_e4m3_encode_matches_torch_rounding():
    rng = np.random.default_rng(7)
    grid = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))  # 0 .. 448
    mids = (grid[:-1] + grid[1:]) / 2                              # ties: to even
    vals = [grid, mids, np.nextafter(mids.astype(np.float32), np.float32(0)),
            np.nextafter(mids.astype(np.float32), np.float32(500)),
            rng.uniform(0, 448, 20000) * np.exp2(rng.integers(-14, 1, 20000)),
            rng.uniform(0, 2.0 ** -6, 5000), np.array([0.0, 2.0 ** -11, 3 * 2.0 ** -11])]
    x = np.concatenate([v.astype(np.float32) for v in vals])
    x = np.concatenate([x, -x])
    assert np.array_equal(oracle.e4m3_encode(x.astype(np.float64)), _torch_e4m3(x))


def test_e4m3_encode_saturates_and_keeps_zero_sign():
    c = oracle.e4m3_encode(np.array([448.0, 460.0, 480.0, 1e30, np.inf, -1e9, -0.0, -2.0 ** -12]))
    assert c.tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x80, 0x80]
    assert oracle.e4m3_encode(np.array([np.nan]))[0] & 0x7F == 0x7F


def test_e4m3_scale_exp_is_the_smallest_power_of_two():
    rng = np.random.default_rng(3)
    amaxes = list(rng.uniform(0, 1, 2000) * np.exp2(rng.integers(-40, 40, 2000)))
    amaxes += [448.0 * 2.0 ** k for k in range(-20, 20)]
    amaxes += [math.nextafter(448.0 * 2.0 ** k, math.inf) for k in range(-5, 5)]
    amaxes += [2.0 ** k for k in range(-30, 30)]
    for a in amaxes:
        E = oracle.e4m3_scale_exp(a)
        assert a <= math.ldexp(448.0, E) and a > math.ldexp(448.0, E - 1), (a, E)
    assert oracle.e4m3_scale_exp(0.0) == 0


def _bf16_rows(rows, cols, seed, scale=0.02):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(rows, cols, generator=g) * scale).bfloat16()
    x[1] = 0                        # an all-zero row
    x[2] *= 1e4                     # a wide row
    x[3, 5] = -3.0                  # one large element: most of the row in subnormals
    return x


def test_quantize_rows_match_torch_conversion():
    x = _bf16_rows(16, 96, seed=11)
    codes, scales = oracle.quantize_e4m3_rows(_bf16_bits(x))
    xd = x.double().numpy()
    for r in range(x.shape[0]):
        amax = np.abs(xd[r]).max()
        f, ex = math.frexp(amax) if amax > 0 else (0.5, 0)
        E = 0 if amax == 0 else (ex - 9 if f <= 0.875 else ex - 8)
        assert scales[r] == math.ldexp(1.0, E)
        assert np.array_equal(codes[r], _torch_e4m3(np.ldexp(xd[r], -E)))
    y = oracle.dequantize_e4m3_rows(codes, scales)
    mx = np.abs(y).max(1) / scales
    nz = np.abs(xd).max(1) > 0
    # amax / scale lies in (224, 448]; rounding may bring it down to 224
    assert ((mx[nz] >= 224) & (mx[nz] <= 448)).all()
    # round to nearest with 3 mantissa bits: |error| <= 2^-4 |x| in the normal
    # range, <= half the subnormal spacing 2^-10 (times the scale) below it
    err = np.abs(y - xd)
    normal = np.abs(xd) >= scales[:, None] * 2.0 ** -6
    assert (err[normal] <= 2.0 ** -4 * np.abs(xd[normal])).all()
    assert (err[~normal] <= (scales[:, None] * 2.0 ** -10 * np.ones_like(xd))[~normal]).all()


def _fp8_grid_rows(rows, cols, seed):
    """Rows whose values are already E4M3 values times the row's scale, with
    the row's largest magnitude hitting a code of (224, 448]: quantisation is
    then lossless."""
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 0x7F, (rows, cols)).astype(np.uint8) | (
        rng.integers(0, 2, (rows, cols)).astype(np.uint8) << 7)
    codes[:, 0] = 0x7A                                   # 320
    E = rng.integers(-14, -4, rows)
    v = oracle.e4m3_decode(codes) * np.exp2(E)[:, None]
    return torch.from_numpy(v).bfloat16()


def test_project_gate_fp8_equals_plain_on_representable_operands():
    rows, M, d, dm = 5, 2, 32, 64
    e = _fp8_grid_rows(rows, dm, 1)
    wk = _fp8_grid_rows(M * d, dm, 2).reshape(M, d, dm)
    wv = _fp8_grid_rows(d, dm, 3)
    g = torch.Generator().manual_seed(4)
    h = torch.randn(rows, M, d, generator=g).bfloat16()
    nq = (1 + 0.1 * torch.randn(M, d, generator=g)).numpy()
    nk = (1 + 0.1 * torch.randn(M, d, generator=g)).numpy()
    args = [_bf16_bits(t) for t in (e, wk, wv)]
    a0, d0, o0 = oracle.project_gate(args[0], args[1], args[2], nq, nk, _bf16_bits(h), 1e-6)
    a1, d1, o1 = oracle.project_gate_fp8(args[0], args[1], args[2], nq, nk, _bf16_bits(h), 1e-6)
    assert np.array_equal(a0, a1) and np.array_equal(d0, d1) and np.array_equal(o0, o1)


def test_project_gate_fp8_against_torch_fp64():
    rows, M, d, dm = 6, 2, 64, 96
    g = torch.Generator().manual_seed(9)
    e = (torch.randn(rows, dm, generator=g) * 0.02).bfloat16()
    wk = (torch.randn(M, d, dm, generator=g) / math.sqrt(dm)).bfloat16()
    wv = (torch.randn(d, dm, generator=g) / math.sqrt(dm)).bfloat16()
    h = torch.randn(rows, M, d, generator=g).bfloat16()
    nq = (1 + 0.1 * torch.randn(M, d, generator=g)).numpy()
    nk = (1 + 0.1 * torch.randn(M, d, generator=g)).numpy()
    alpha, delta, out = oracle.project_gate_fp8(_bf16_bits(e), _bf16_bits(wk), _bf16_bits(wv),
                                                nq, nk, _bf16_bits(h), 1e-6)

    def deq(x):  # per row: power-of-two scale from frexp, codes by torch's conversion
        x = x.double().reshape(-1, x.shape[-1])
        amax = x.abs().amax(1)
        out = torch.empty_like(x)
        for r in range(x.shape[0]):
            f, ex = math.frexp(float(amax[r]))
            E = 0 if amax[r] == 0 else (ex - 9 if f <= 0.875 else ex - 8)
            q = torch.from_numpy(np.ldexp(x[r].numpy(), -E)).float().to(torch.float8_e4m3fn)
            out[r] = q.double() * 2.0 ** E
        return out

    E8, WV8 = deq(e), deq(wv)
    WK8 = deq(wk).reshape(M, d, dm)
    H = h.double()
    k = torch.einsum("rj,mij->rmi", E8, WK8)
    v = E8 @ WV8.T
    qn = H / torch.sqrt(H.pow(2).mean(-1, keepdim=True) + 1e-6) * torch.from_numpy(nq).double()
    kn = k / torch.sqrt(k.pow(2).mean(-1, keepdim=True) + 1e-6) * torch.from_numpy(nk).double()
    a_ref = torch.sigmoid((qn * kn).sum(-1) / math.sqrt(d))
    assert np.allclose(alpha, a_ref.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(delta, (a_ref[..., None] * v[:, None, :]).numpy(), rtol=1e-12, atol=1e-12)
    # and it differs from the bf16 projection by quantisation error only
    a0, d0, _ = oracle.project_gate(_bf16_bits(e), _bf16_bits(wk), _bf16_bits(wv), nq, nk,
                                    _bf16_bits(h), 1e-6)
    rel = np.linalg.norm(delta - d0) / np.linalg.norm(d0)
    assert 1e-4 < rel < 0.1


# ------------------------------------------------------- backward (row f4)

def _bw_problem(R=3, M=2, d=8, dm=12, seed=0):
    rng = np.random.default_rng(seed)
    e = rng.normal(size=(R, dm))
    wk = rng.normal(size=(M, d, dm)) / 3
    wv = rng.normal(size=(d, dm)) / 3
    h = rng.normal(size=(R, M, d))
    g = rng.normal(size=(R, M, d))
    nq = (1 + 0.1 * rng.normal(size=(M, d))).astype(np.float32)
    nk = (1 + 0.1 * rng.normal(size=(M, d))).astype(np.float32)
    return e, wk, wv, nq, nk, h, g


def _loss(e, wk, wv, nq, nk, h, g):
    _, delta, _ = oracle.project_gate_mixed(e, wk, wv, nq, nk, h, 1e-6)
    return float(np.sum(g * (h + delta)))


def test_backward_matches_finite_differences():
    e, wk, wv, nq, nk, h, g = _bw_problem()
    b = oracle.backward(e, wk, wv, nq, nk, h, g, 1e-6)
    step = 1e-6
    for name, arr, grad in (("e", e, b["de"]), ("w_k", wk, b["dw_k"]), ("w_v", wv, b["dw_v"]),
                            ("h", h, b["dh"])):
        rng = np.random.default_rng(len(name))
        for flat in rng.choice(arr.size, size=min(arr.size, 12), replace=False):
            idx = np.unravel_index(flat, arr.shape)
            orig = arr[idx]
            arr[idx] = orig + step
            lp = _loss(e, wk, wv, nq, nk, h, g)
            arr[idx] = orig - step
            lm = _loss(e, wk, wv, nq, nk, h, g)
            arr[idx] = orig
            fd = (lp - lm) / (2 * step)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, grad[idx])


def test_backward_matches_torch_autograd():
    e, wk, wv, nq, nk, h, g = _bw_problem(R=4, M=3, d=16, dm=24, seed=5)
    b = oracle.backward(e, wk, wv, nq, nk, h, g, 1e-6)
    E, WK, WV, H = [torch.tensor(x, requires_grad=True) for x in (e, wk, wv, h)]
    NQ = torch.tensor(nq.astype(np.float64), requires_grad=True)
    NK = torch.tensor(nk.astype(np.float64), requires_grad=True)
    k = torch.einsum("rj,mij->rmi", E, WK)
    v = E @ WV.T
    qn = torch.nn.functional.rms_norm(H, (16,), eps=1e-6) * NQ
    kn = torch.nn.functional.rms_norm(k, (16,), eps=1e-6) * NK
    a = torch.sigmoid((qn * kn).sum(-1) / 4.0)
    out = H + a[..., None] * v[:, None, :]
    (out * torch.tensor(g)).sum().backward()
    for mine, ref in ((b["de"], E.grad), (b["dw_k"], WK.grad), (b["dw_v"], WV.grad),
                      (b["dh"], H.grad), (b["dnorm_q"], NQ.grad), (b["dnorm_k"], NK.grad)):
        assert np.allclose(mine, ref.numpy(), rtol=1e-10, atol=1e-12)


def test_backward_special_cases():
    e, wk, wv, nq, nk, h, g = _bw_problem(seed=2)
    z = oracle.backward(e, wk, wv, nq, nk, h, np.zeros_like(g), 1e-6)
    assert all((v == 0).all() for k, v in z.items() if k != "dh") and (z["dh"] == 0).all()
    # W_V = 0: alpha multiplies nothing, so dalpha = 0 and only the residual and dv remain
    b = oracle.backward(e, wk, np.zeros_like(wv), nq, nk, h, g, 1e-6)
    assert np.array_equal(b["dh"], g) and (b["dw_k"] == 0).all() and (b["dnorm_q"] == 0).all()
    alpha, _, _ = oracle.project_gate_mixed(e, wk, np.zeros_like(wv), nq, nk, h, 1e-6)
    dv = np.einsum("rm,rmi->ri", alpha, g)
    assert np.allclose(b["dw_v"], dv.T @ e, rtol=1e-12, atol=1e-14)


def test_backward_bf16_rounding_of_gemm_operands():
    e, wk, wv, nq, nk, h, g = _bw_problem(R=5, M=2, d=16, dm=24, seed=7)
    exact = oracle.backward(e, wk, wv, nq, nk, h, g, 1e-6)
    b = oracle.backward(e, wk, wv, nq, nk, h, g, 1e-6, round_dkv=True)
    want = torch.tensor(exact["dkv"]).float().bfloat16().double().numpy()
    assert np.array_equal(b["dkv"], want)
    assert np.array_equal(b["dh"], exact["dh"]) and np.array_equal(b["dnorm_q"], exact["dnorm_q"])
    M, d, dm = wk.shape
    dw = torch.tensor(want).T @ torch.tensor(e)
    assert np.allclose(np.concatenate([b["dw_k"].reshape(M * d, dm), b["dw_v"]]), dw.numpy(),
                       rtol=1e-12, atol=1e-14)
    W = np.concatenate([wk.reshape(M * d, dm), wv])
    assert np.allclose(b["de"], want @ W, rtol=1e-12, atol=1e-14)


def test_table_grad_matches_numpy_scatter_add():
    rng = np.random.default_rng(4)
    rows, S, dh = 50, 3, 4
    sizes = [7, 11, 13]
    z = np.stack([rng.integers(0, p, rows) for p in sizes], 1)   # repeats: rows collide
    de = rng.normal(size=(rows, S * dh))
    got = oracle.table_grad(de, z, sizes, dh)
    for s, p in enumerate(sizes):
        want = np.zeros((p, dh))
        np.add.at(want, z[:, s], de[:, s * dh:(s + 1) * dh])
        assert np.allclose(got[s], want, rtol=1e-14, atol=1e-15)
