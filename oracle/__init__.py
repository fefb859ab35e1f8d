"""CPU oracle for the Engram lookup-and-gate forward.

TEST INFRASTRUCTURE ONLY.  The tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  The product path never
imports this package, and this package never imports the product package:
they share no code.

The arithmetic lives in ``engram_oracle.c`` (plain single-threaded C, double
accumulation); this module only marshals numpy arrays through ctypes and
chains the steps in the paper's order ("Conditional Memory via Scalable
Lookup", section 2.2-2.4).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "engram_oracle.c")
_LIB = os.path.join(_HERE, "_engram_oracle.so")

F32, BF16, F64 = 0, 1, 2
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, no fast-math) into an in-tree .so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fno-fast-math",
                               "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i32, i64, u64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_double
        L.eo_splitmix64_next.argtypes = [P]
        L.eo_splitmix64_next.restype = u64
        L.eo_hash_multipliers.argtypes = [u64, i32, i32, P]
        L.eo_hash_multipliers.restype = None
        L.eo_is_prime.argtypes = [i64]
        L.eo_is_prime.restype = ctypes.c_int
        L.eo_table_primes.argtypes = [i64, i32, P]
        L.eo_table_primes.restype = ctypes.c_int
        L.eo_compress.argtypes = [P, i64, P, i32, P]
        L.eo_compress.restype = i64
        L.eo_hash.argtypes = [P, i32, i32, i32, i32, i32, P, i32, P, i32, P, P]
        L.eo_hash.restype = None
        L.eo_gather.argtypes = [P, i32, i32, P, i64, i32, P]
        L.eo_gather.restype = None
        L.eo_project.argtypes = [P, i32, i64, i32, P, i32, P]
        L.eo_project.restype = None
        L.eo_gate.argtypes = [P, P, P, P, i32, f64]
        L.eo_gate.restype = f64
        L.eo_project_gate.argtypes = [P, i32, i64, i32, P, P, P, P, i32, i32, f64, P,
                                      P, P, P, P, P, P]
        L.eo_project_gate.restype = None
        L.eo_short_conv_at.argtypes = [P, P, i32, i32, P, P, f64, P, P]
        L.eo_short_conv_at.restype = None
        L.eo_short_conv.argtypes = [P, i32, i32, P, i32, i32, P, f64, P, P, P, P]
        L.eo_short_conv.restype = None
        L.eo_add_round.argtypes = [P, i32, i64, P, P]
        L.eo_add_round.restype = None
        L.eo_project_gate_mixed.argtypes = [P, i32, i64, i32, P, P, P, P, i32, i32, f64, P,
                                            i32, P, P, P, P, P, P]
        L.eo_project_gate_mixed.restype = None
        L.eo_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.eo_e4m3_decode.restype = f64
        L.eo_e4m3_encode.argtypes = [f64]
        L.eo_e4m3_encode.restype = ctypes.c_uint8
        L.eo_e4m3_scale_exp.argtypes = [f64]
        L.eo_e4m3_scale_exp.restype = i32
        L.eo_quantize_e4m3_rows.argtypes = [P, i32, i64, i32, P, P]
        L.eo_quantize_e4m3_rows.restype = None
        L.eo_dequantize_e4m3_rows.argtypes = [P, P, i64, i32, P]
        L.eo_dequantize_e4m3_rows.restype = None
        L.eo_backward.argtypes = [P, i32, i64, i32, P, P, P, P, i32, i32, f64, P, i32, P, i32,
                                  P, P, P, P, P, P, P, P, P]
        L.eo_backward.restype = None
        L.eo_table_grad.argtypes = [P, P, i64, i32, i32, P]
        L.eo_table_grad.restype = None
        _lib = L
    return _lib


def _dtype_of(a: np.ndarray) -> int:
    return {np.dtype(np.float64): F64, np.dtype(np.float32): F32,
            np.dtype(np.uint16): BF16}[a.dtype]


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


# ----------------------------------------------------------------- generators

def splitmix64_stream(seed: int, n: int) -> list:
    st = np.array([seed & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64)
    return [int(lib().eo_splitmix64_next(_p(st))) for _ in range(n)]


def hash_multipliers(seed: int, num_tables: int, max_order: int) -> np.ndarray:
    m = np.zeros((num_tables, max_order), dtype=np.uint64)
    lib().eo_hash_multipliers(seed & 0xFFFFFFFFFFFFFFFF, num_tables, max_order, _p(m))
    return m


def is_prime(n: int) -> bool:
    return bool(lib().eo_is_prime(int(n)))


def table_primes(target: int, num_tables: int) -> np.ndarray:
    p = np.zeros(num_tables, dtype=np.int64)
    if lib().eo_table_primes(int(target), num_tables, _p(p)) != 0:
        raise ValueError("prime target must be >= 2")
    return p


# --------------------------------------------------------------------- steps

def compress(tokens: np.ndarray, comp_map: np.ndarray) -> np.ndarray:
    """x' = P(x) (section 2.2).  Raises on tokens outside [0, V)."""
    x = np.ascontiguousarray(tokens, dtype=np.int32)
    m = np.ascontiguousarray(comp_map, dtype=np.int32)
    c = np.empty_like(x)
    bad = lib().eo_compress(_p(x), x.size, _p(m), m.size, _p(c))
    if bad:
        raise ValueError("%d tokens outside [0, V)" % bad)
    return c


def hash_indices(c: np.ndarray, pad: int, orders: Sequence[int], heads: int,
                 mult: np.ndarray, primes: np.ndarray, t_begin: int = 0) -> np.ndarray:
    """z [B*(T-t_begin), S] int64 (Eq. 1)."""
    c = np.ascontiguousarray(c, dtype=np.int32)
    B, T = c.shape
    o = np.ascontiguousarray(orders, dtype=np.int32)
    mult = np.ascontiguousarray(mult, dtype=np.uint64)
    primes = np.ascontiguousarray(primes, dtype=np.int64)
    S = len(o) * heads
    assert mult.shape[0] == S and primes.shape[0] == S and mult.shape[1] >= max(o)
    z = np.empty((B * (T - t_begin), S), dtype=np.int64)
    lib().eo_hash(_p(c), B, T, t_begin, pad, len(o), _p(o), heads, _p(mult), mult.shape[1],
                  _p(primes), _p(z))
    return z


def gather(tables: Sequence[np.ndarray], z: np.ndarray) -> np.ndarray:
    """e [rows, S*d_h] (Eq. 2): byte copies of the addressed rows.

    Tables are numpy arrays of float32 or uint16 (bf16 bit patterns)."""
    z = np.ascontiguousarray(z, dtype=np.int64)
    rows, S = z.shape
    assert len(tables) == S
    t0 = tables[0]
    d_h = t0.shape[1]
    for s, t in enumerate(tables):
        assert t.flags["C_CONTIGUOUS"] and t.dtype == t0.dtype and t.shape[1] == d_h
        if z.size and (z[:, s].min() < 0 or z[:, s].max() >= t.shape[0]):
            raise IndexError("index outside table %d" % s)
    ptrs = (ctypes.c_void_p * S)(*[t.ctypes.data for t in tables])
    e = np.empty((rows, S * d_h), dtype=t0.dtype)
    lib().eo_gather(ptrs, t0.itemsize, d_h, _p(z), rows, S, _p(e))
    return e


def project(e: np.ndarray, w: np.ndarray) -> np.ndarray:
    """y = e W^T in double (Eq. 3).  w is [n_out, d_mem]."""
    dtype = F32 if e.dtype == np.float32 else BF16
    assert w.dtype == e.dtype
    e = np.ascontiguousarray(e)
    w = np.ascontiguousarray(w)
    rows, dm = e.shape
    y = np.empty((rows, w.shape[0]), dtype=np.float64)
    lib().eo_project(_p(e), dtype, rows, dm, _p(w), w.shape[0], _p(y))
    return y


def gate(h: np.ndarray, k: np.ndarray, wq: np.ndarray, wk: np.ndarray, eps: float) -> float:
    """alpha of one position and branch (Eq. 4), from double h and k."""
    h = np.ascontiguousarray(h, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    wq = np.ascontiguousarray(wq, dtype=np.float32)
    wk = np.ascontiguousarray(wk, dtype=np.float32)
    return float(lib().eo_gate(_p(h), _p(k), _p(wq), _p(wk), h.shape[0], eps))


def project_gate(e, w_k, w_v, norm_q, norm_k, h, eps: float, want_delta: bool = True):
    """alpha [rows, M], delta [rows, M, d] (double), out [rows, M, d] (h's dtype).

    Eq. (3), Eq. (4)/(6) and the gated residual, for rows whose e is given."""
    dtype = F32 if e.dtype == np.float32 else BF16
    e = np.ascontiguousarray(e)
    rows, dm = e.shape
    M, d, dm2 = w_k.shape
    assert dm2 == dm and w_v.shape == (d, dm) and h.shape == (rows, M, d)
    assert w_k.dtype == e.dtype == w_v.dtype == h.dtype
    w_k = np.ascontiguousarray(w_k)
    w_v = np.ascontiguousarray(w_v)
    h = np.ascontiguousarray(h)
    nq = np.ascontiguousarray(norm_q, dtype=np.float32)
    nk = np.ascontiguousarray(norm_k, dtype=np.float32)
    alpha = np.empty((rows, M), dtype=np.float64)
    delta = np.empty((rows, M, d), dtype=np.float64) if want_delta else None
    out = np.empty_like(h)
    kb = np.empty(M * d, dtype=np.float64)
    vb = np.empty(d, dtype=np.float64)
    hb = np.empty(d, dtype=np.float64)
    lib().eo_project_gate(_p(e), dtype, rows, dm, _p(w_k), _p(w_v), _p(nq), _p(nk), M, d, eps,
                          _p(h), _p(alpha), _p(delta) if delta is not None else None, _p(out),
                          _p(kb), _p(vb), _p(hb))
    return alpha, delta, out


# ------------------------------------------------------------ FP8 projection

def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Values (double) of E4M3 codes (NaN for S.1111.111)."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    L = lib()
    return np.array([L.eo_e4m3_decode(int(v)) for v in c.ravel()]).reshape(c.shape)


def e4m3_encode(y: np.ndarray) -> np.ndarray:
    """E4M3 codes of y: nearest, ties to even, saturating at +-448."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    L = lib()
    return np.array([L.eo_e4m3_encode(float(v)) for v in y.ravel()],
                    dtype=np.uint8).reshape(y.shape)


def e4m3_scale_exp(amax: float) -> int:
    """Smallest E with amax <= 448 * 2^E (0 for amax = 0)."""
    return int(lib().eo_e4m3_scale_exp(float(amax)))


def quantize_e4m3_rows(x: np.ndarray):
    """(codes uint8 [rows, cols], scales float32 [rows]) of x [rows, cols]
    (float32, or uint16 bf16 bit patterns): one power-of-two scale per row."""
    x = np.ascontiguousarray(x)
    dtype = F32 if x.dtype == np.float32 else BF16
    assert x.dtype in (np.float32, np.uint16) and x.ndim == 2
    rows, cols = x.shape
    codes = np.empty((rows, cols), dtype=np.uint8)
    scales = np.empty(rows, dtype=np.float32)
    lib().eo_quantize_e4m3_rows(_p(x), dtype, rows, cols, _p(codes), _p(scales))
    return codes, scales


def dequantize_e4m3_rows(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    rows, cols = codes.shape
    y = np.empty((rows, cols), dtype=np.float64)
    lib().eo_dequantize_e4m3_rows(_p(codes), _p(scales), rows, cols, _p(y))
    return y


def project_gate_mixed(e, w_k, w_v, norm_q, norm_k, h, eps: float, want_delta: bool = True):
    """project_gate with e, w_k, w_v in double and h in its own dtype (float64,
    float32 or uint16 bf16 bits; out in the same)."""
    e = np.ascontiguousarray(e, dtype=np.float64)
    rows, dm = e.shape
    M, d, dm2 = w_k.shape
    assert dm2 == dm and w_v.shape == (d, dm) and h.shape == (rows, M, d)
    w_k = np.ascontiguousarray(w_k, dtype=np.float64)
    w_v = np.ascontiguousarray(w_v, dtype=np.float64)
    h = np.ascontiguousarray(h)
    hdtype = _dtype_of(h)
    nq = np.ascontiguousarray(norm_q, dtype=np.float32)
    nk = np.ascontiguousarray(norm_k, dtype=np.float32)
    alpha = np.empty((rows, M), dtype=np.float64)
    delta = np.empty((rows, M, d), dtype=np.float64) if want_delta else None
    out = np.empty_like(h)
    kb = np.empty(M * d, dtype=np.float64)
    vb = np.empty(d, dtype=np.float64)
    hb = np.empty(d, dtype=np.float64)
    lib().eo_project_gate_mixed(_p(e), F64, rows, dm, _p(w_k), _p(w_v), _p(nq), _p(nk), M, d,
                                eps, _p(h), hdtype, _p(alpha),
                                _p(delta) if delta is not None else None, _p(out),
                                _p(kb), _p(vb), _p(hb))
    return alpha, delta, out


def quantize_weights_e4m3(w_k: np.ndarray, w_v: np.ndarray):
    """Dequantised W_K [M, d, d_mem] and W_V [d, d_mem]: one scale per output
    channel (row of W)."""
    M, d, dm = w_k.shape
    wk = dequantize_e4m3_rows(*quantize_e4m3_rows(np.ascontiguousarray(w_k).reshape(M * d, dm)))
    wv = dequantize_e4m3_rows(*quantize_e4m3_rows(np.ascontiguousarray(w_v)))
    return wk.reshape(M, d, dm), wv


def project_gate_fp8(e, w_k, w_v, norm_q, norm_k, h, eps: float, want_delta: bool = True,
                     weights=None):
    """The FP8 form of project_gate (section 2.4): e quantised per row, W per
    output channel, then Eq. (3)-(4)/(6) on the dequantised operands.
    `weights` may hold quantize_weights_e4m3's result to skip recomputing it."""
    ehat = dequantize_e4m3_rows(*quantize_e4m3_rows(e))
    wk, wv = weights if weights is not None else quantize_weights_e4m3(w_k, w_v)
    return project_gate_mixed(ehat, wk, wv, norm_q, norm_k, h, eps, want_delta)


# ------------------------------------------------------------------ backward

def backward(e, w_k, w_v, norm_q, norm_k, h, dout, eps: float, round_dkv: bool = False):
    """Gradients of project_gate's out for the upstream gradient dout [rows, M, d].

    e, w_k, w_v share one dtype (float64, float32 or uint16 bf16 bits); h has
    its own.  Returns dict(dh [rows, M, d], dkv [rows, (M+1) d] (dk of each
    branch, then dv; bf16-rounded when round_dkv), dw_k [M, d, d_mem],
    dw_v [d, d_mem], dnorm_q [M, d], dnorm_k [M, d], de [rows, d_mem]), all
    double."""
    e = np.ascontiguousarray(e)
    rows, dm = e.shape
    M, d, dm2 = w_k.shape
    assert dm2 == dm and w_v.shape == (d, dm) and h.shape == (rows, M, d)
    w_k = np.ascontiguousarray(w_k, dtype=e.dtype)
    w_v = np.ascontiguousarray(w_v, dtype=e.dtype)
    h = np.ascontiguousarray(h)
    g = np.ascontiguousarray(dout, dtype=np.float64)
    assert g.shape == h.shape
    nq = np.ascontiguousarray(norm_q, dtype=np.float32)
    nk = np.ascontiguousarray(norm_k, dtype=np.float32)
    dh = np.empty((rows, M, d))
    dkv = np.empty((rows, (M + 1) * d))
    dw = np.zeros(((M + 1) * d, dm))
    dwq = np.zeros((M, d))
    dwk = np.zeros((M, d))
    de = np.empty((rows, dm))
    kb, vb, hb = np.empty(M * d), np.empty(d), np.empty(d)
    lib().eo_backward(_p(e), _dtype_of(e), rows, dm, _p(w_k), _p(w_v), _p(nq), _p(nk), M, d,
                      eps, _p(h), _dtype_of(h), _p(g), 1 if round_dkv else 0, _p(dh), _p(dkv),
                      _p(dw), _p(dwq), _p(dwk), _p(de), _p(kb), _p(vb), _p(hb))
    return dict(dh=dh, dkv=dkv, dw_k=dw[:M * d].reshape(M, d, dm), dw_v=dw[M * d:],
                dnorm_q=dwq, dnorm_k=dwk, de=de)


def table_grad(de: np.ndarray, z: np.ndarray, table_rows: Sequence[int], d_head: int):
    """dE_s [p_s, d_h] (double) += the slot-s slices of de at rows z[:, s] (Eq. 2
    transposed); returns the list of S arrays."""
    de = np.ascontiguousarray(de, dtype=np.float64)
    z = np.ascontiguousarray(z, dtype=np.int64)
    rows, S = z.shape
    assert de.shape == (rows, S * d_head) and len(table_rows) == S
    if z.size:
        assert (z >= 0).all() and (z < np.asarray(table_rows)[None, :]).all()
    out = [np.zeros((int(p), d_head)) for p in table_rows]
    ptrs = (ctypes.c_void_p * S)(*[t.ctypes.data for t in out])
    lib().eo_table_grad(_p(de), _p(z), rows, S, d_head, ptrs)
    return out


# ---------------------------------------------------------------- short conv

def short_conv(vt: np.ndarray, conv_w: np.ndarray, norm_w: np.ndarray, dil: int,
               eps: float) -> np.ndarray:
    """Y = SiLU(Conv1D(RMSNorm(V~))) + V~ over one sequence (Eq. 5).

    vt [n_pos, d] gated values of one branch; conv_w [d, W] (tap i multiplies
    position t - i*dil); norm_w [d].  Returns Y [n_pos, d] in double."""
    vt = np.ascontiguousarray(vt, dtype=np.float64)
    n_pos, d = vt.shape
    cw = np.ascontiguousarray(conv_w, dtype=np.float32)
    nw = np.ascontiguousarray(norm_w, dtype=np.float32)
    W = cw.shape[1]
    assert cw.shape == (d, W) and nw.shape == (d,)
    y = np.empty_like(vt)
    taps = np.empty(W * d, dtype=np.float64)
    have = np.empty(W, dtype=np.int32)
    norm = np.empty(d, dtype=np.float64)
    lib().eo_short_conv(_p(vt), n_pos, d, _p(cw), W, dil, _p(nw), eps, _p(y), _p(taps),
                        _p(have), _p(norm))
    return y


def short_conv_at(taps: np.ndarray, have: np.ndarray, conv_w: np.ndarray, norm_w: np.ndarray,
                  eps: float) -> np.ndarray:
    """Y at one position (Eq. 5) from V~ at positions t - i*dil (taps [W, d];
    have[i] = 0 where the position precedes the sequence)."""
    taps = np.ascontiguousarray(taps, dtype=np.float64)
    W, d = taps.shape
    have = np.ascontiguousarray(have, dtype=np.int32)
    cw = np.ascontiguousarray(conv_w, dtype=np.float32)
    nw = np.ascontiguousarray(norm_w, dtype=np.float32)
    y = np.empty(d, dtype=np.float64)
    norm = np.empty(d, dtype=np.float64)
    lib().eo_short_conv_at(_p(taps), _p(have), W, d, _p(cw), _p(nw), eps, _p(y), _p(norm))
    return y


def add_round(h: np.ndarray, y: np.ndarray) -> np.ndarray:
    """h + y rounded to h's dtype (fp32, or bf16 bits as uint16)."""
    h = np.ascontiguousarray(h)
    y = np.ascontiguousarray(y, dtype=np.float64)
    assert y.size == h.size
    out = np.empty_like(h)
    lib().eo_add_round(_p(h), F32 if h.dtype == np.float32 else BF16, h.size, _p(y), _p(out))
    return out


# ------------------------------------------------------------------ pipeline

def forward_indices(tokens: np.ndarray, comp_map: np.ndarray, cvocab: int, orders, heads: int,
                    hash_seed: int, rows_target: int, t_begin: int = 0,
                    pad: Optional[int] = None):
    """Compress, form n-grams and hash: returns (c, z, mult, primes)."""
    S = len(orders) * heads
    mult = hash_multipliers(hash_seed, S, max(orders))
    primes = table_primes(rows_target, S)
    c = compress(tokens, comp_map)
    z = hash_indices(c, cvocab if pad is None else pad, orders, heads, mult, primes, t_begin)
    return c, z, mult, primes
