"""Thin ctypes binding of libengram.so (include/engram.h).

Argument marshalling only: every step of the forward runs in the library's
CUDA kernels.  Functions keep the C names; ``Engram`` wraps a handle and
accepts torch tensors (device memory, streams) and passes their pointers.
There is no CPU fallback: if the library is missing, importing this module
raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libengram.so")

ENGRAM_F32, ENGRAM_BF16 = 0, 1
ENGRAM_DEVICE, ENGRAM_PINNED_HOST = 0, 1
ENGRAM_OK, ENGRAM_ERR_INVALID, ENGRAM_ERR_BOUNDS, ENGRAM_ERR_CUDA = 0, 1, 2, 3
ENGRAM_ERR_OOM, ENGRAM_ERR_TIMEOUT, ENGRAM_ERR_UNSUPPORTED, ENGRAM_ERR_STATE = 4, 5, 6, 7
MAX_ORDERS, MAX_TABLES, MAX_BRANCHES, MAX_SHARDS = 4, 64, 4, 8
IPC_HANDLE_BYTES = 64
ENGRAM_FLAG_NO_CTA_PAIRS = 1
ENGRAM_FLAG_NO_FUSED_SHORT = 2
ENGRAM_PREFETCH_HOST_THREADS, ENGRAM_PREFETCH_ZERO_COPY = 0, 1

#: every symbol include/engram.h declares
EXPORTS = ("engram_create", "engram_destroy", "engram_config_size", "engram_last_error",
           "engram_set_params", "engram_reserve", "engram_get_hash_params", "engram_hash",
           "engram_gather", "engram_forward", "engram_prefetch", "engram_check_errors",
           "engram_profile_next_forward", "engram_kernel_launches",
           "engram_project_gate_noalloc", "engram_selftest_timeout", "engram_set_short_conv",
           "engram_build_hot_cache", "engram_prefetch_hot_hits", "engram_set_fp8",
           "engram_quantize_e4m3", "engram_backward", "engram_profile_next_backward",
           "engram_set_prefetch", "engram_set_table_shards", "engram_ipc_handle",
           "engram_ipc_open", "engram_ipc_close", "engram_prefetch_wait",
           "engram_forward_host", "engram_backward_host")


class engram_config(ctypes.Structure):
    _fields_ = [
        ("vocab", ctypes.c_int32), ("cvocab", ctypes.c_int32), ("pad_id", ctypes.c_int32),
        ("num_orders", ctypes.c_int32), ("orders", ctypes.c_int32 * MAX_ORDERS),
        ("heads", ctypes.c_int32), ("d_head", ctypes.c_int32), ("d_hidden", ctypes.c_int32),
        ("branches", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("table_location", ctypes.c_int32), ("eps", ctypes.c_float),
        ("flags", ctypes.c_int32), ("table_rows_target", ctypes.c_int64),
        ("hash_seed", ctypes.c_uint64), ("primes", ctypes.c_int64 * MAX_TABLES),
        ("comp_map", ctypes.POINTER(ctypes.c_int32)),
    ]


class EngramError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__("engram error %d: %s" % (code, msg))
        self.code = code


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError("libengram.so is not built (run hashed_gram_embedding_compress_b200."
                          "build.build() or __graft_entry__.build()); there is no fallback")
    L = ctypes.CDLL(LIB_PATH)
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    H = ctypes.c_void_p
    sig = {
        "engram_create": ([ctypes.POINTER(engram_config), ctypes.POINTER(H)], ctypes.c_int),
        "engram_destroy": ([H], None),
        "engram_config_size": ([], ctypes.c_size_t),
        "engram_last_error": ([H], ctypes.c_char_p),
        "engram_set_params": ([H, P, P, P, P, P], ctypes.c_int),
        "engram_reserve": ([H, i64], ctypes.c_int),
        "engram_set_short_conv": ([H, P, P, i32, i32, P], ctypes.c_int),
        "engram_build_hot_cache": ([H, P, i32, i32, i32, i64, P], ctypes.c_int),
        "engram_prefetch_hot_hits": ([H, P], ctypes.c_int),
        "engram_set_fp8": ([H, i32, P], ctypes.c_int),
        "engram_quantize_e4m3": ([H, P, i64, i32, P, P, P], ctypes.c_int),
        "engram_backward": ([H, P, P, i32, i32, i32, P, P, P, P, P, P, P, P, P], ctypes.c_int),
        "engram_get_hash_params": ([H, P, P], ctypes.c_int),
        "engram_hash": ([H, P, i32, i32, i32, P, P], ctypes.c_int),
        "engram_gather": ([H, P, i64, P, P], ctypes.c_int),
        "engram_forward": ([H, P, P, i32, i32, i32, P, P, P, P, P], ctypes.c_int),
        "engram_forward_host": ([H, P, i32, i32, i32, P, P, P, P], ctypes.c_int),
        "engram_backward_host": ([H, P, i32, i32, i32, P, P, P, P, P, P, P, P, P],
                                 ctypes.c_int),
        "engram_prefetch": ([H, P, i32, i32, i32, P, P], ctypes.c_int),
        "engram_set_prefetch": ([H, i32, i32], ctypes.c_int),
        "engram_prefetch_wait": ([H], ctypes.c_int),
        "engram_set_table_shards": ([H, i32, P], ctypes.c_int),
        "engram_ipc_handle": ([H, P, P], ctypes.c_int),
        "engram_ipc_open": ([H, P, P], ctypes.c_int),
        "engram_ipc_close": ([H, P], ctypes.c_int),
        "engram_check_errors": ([H, P], ctypes.c_int),
        "engram_profile_next_forward": ([H, P, i32], ctypes.c_int),
        "engram_profile_next_backward": ([H, P, i32], ctypes.c_int),
        "engram_kernel_launches": ([H], ctypes.c_int64),
        "engram_project_gate_noalloc": ([H, P, i64, P, P, P, P], ctypes.c_int),
        "engram_selftest_timeout": ([H, P], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    if L.engram_config_size() != ctypes.sizeof(engram_config):
        raise ImportError("engram_config layout mismatch between binding and library")
    return L


lib = _load()


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream_ptr(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def make_config(*, vocab, cvocab, comp_map: torch.Tensor, orders: Sequence[int] = (2, 3),
                heads=8, d_head=80, d_hidden=2560, branches=1, dtype="bf16", eps=1e-6,
                table_rows_target=1 << 20, primes: Optional[Sequence[int]] = None,
                hash_seed=0, pad_id=-1, table_location="device", flags=0):
    """Fill an engram_config; keeps the host map alive on the returned object."""
    c = engram_config()
    c.vocab, c.cvocab, c.pad_id = vocab, cvocab, pad_id
    c.num_orders = len(orders)
    for i, o in enumerate(orders):
        c.orders[i] = o
    c.heads, c.d_head, c.d_hidden, c.branches = heads, d_head, d_hidden, branches
    c.dtype = {"f32": ENGRAM_F32, "bf16": ENGRAM_BF16}[dtype]
    c.table_location = {"device": ENGRAM_DEVICE, "pinned_host": ENGRAM_PINNED_HOST}[table_location]
    c.eps = eps
    c.flags = flags
    c.table_rows_target = table_rows_target
    c.hash_seed = hash_seed & 0xFFFFFFFFFFFFFFFF
    if primes is not None:
        for i, p in enumerate(primes):
            c.primes[i] = p
    m = comp_map.to(torch.int32).contiguous().cpu()
    c._map_keepalive = m
    c.comp_map = ctypes.cast(m.data_ptr(), ctypes.POINTER(ctypes.c_int32))
    return c


class Engram:
    """One handle of the forward lookup-and-gate module."""

    def __init__(self, cfg: engram_config):
        self._h = ctypes.c_void_p()
        rc = lib.engram_create(ctypes.byref(cfg), ctypes.byref(self._h))
        if rc != ENGRAM_OK:
            raise EngramError(rc, lib.engram_last_error(None).decode())
        self.cfg = cfg
        self.S = cfg.num_orders * cfg.heads
        self.max_order = cfg.orders[cfg.num_orders - 1]
        self.d_mem = self.S * cfg.d_head
        self._params = None

    def _check(self, rc):
        if rc != ENGRAM_OK:
            raise EngramError(rc, lib.engram_last_error(self._h).decode())

    def close(self):
        if self._h:
            lib.engram_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # --------------------------------------------------------------- calls
    def hash_params(self):
        primes = torch.zeros(self.S, dtype=torch.int64)
        mult = torch.zeros(self.S * self.max_order, dtype=torch.int64)
        self._check(lib.engram_get_hash_params(self._h, primes.data_ptr(), mult.data_ptr()))
        return primes, mult.view(self.S, self.max_order)

    def set_params(self, tables: Sequence[torch.Tensor], w_k, w_v, norm_q, norm_k):
        arr = (ctypes.c_void_p * self.S)(*[t.data_ptr() for t in tables])
        self._check(lib.engram_set_params(self._h, ctypes.cast(arr, ctypes.c_void_p), _ptr(w_k),
                                          _ptr(w_v), _ptr(norm_q), _ptr(norm_k)))
        self._params = (list(tables), w_k, w_v, norm_q, norm_k)  # borrowed: keep alive

    def set_short_conv(self, conv_w, norm_w, kernel_size: int = 4, dilation: int = 3,
                       stream=None):
        """Switch on the short convolution of Eq. (5) with conv_w [d, kernel_size]
        and norm_w [d] (fp32, device; copied); kernel_size 0 switches it off."""
        self._check(lib.engram_set_short_conv(self._h, _ptr(conv_w), _ptr(norm_w), kernel_size,
                                              dilation, _stream_ptr(stream)))

    def set_table_shards(self, shards):
        """Row-sharded tables: shards[s][j] = shard j of table s (a tensor, or a
        device pointer as int), row z of table s at local row z // N of shard
        z % N."""
        N = len(shards[0])
        flat = [x for row in shards for x in row]
        if len(shards) != self.S or any(len(row) != N for row in shards):
            raise EngramError(ENGRAM_ERR_INVALID, "shards must be S lists of N entries")
        arr = (ctypes.c_void_p * len(flat))(*[_ptr(x) for x in flat])
        self._check(lib.engram_set_table_shards(self._h, N, ctypes.cast(arr, ctypes.c_void_p)))
        self._shards = flat  # borrowed: keep alive

    def ipc_handle(self, t) -> bytes:
        """Inter-process handle of the allocation that starts at t (64 bytes)."""
        buf = ctypes.create_string_buffer(IPC_HANDLE_BYTES)
        self._check(lib.engram_ipc_handle(self._h, _ptr(t), buf))
        return buf.raw

    def ipc_open(self, handle: bytes) -> int:
        """Map another process's allocation; returns its device pointer here."""
        p = ctypes.c_void_p()
        self._check(lib.engram_ipc_open(self._h, ctypes.c_char_p(handle), ctypes.byref(p)))
        return p.value

    def ipc_close(self, ptr: int):
        self._check(lib.engram_ipc_close(self._h, ptr))

    def set_fp8(self, enable: bool = True, stream=None):
        """Projections on E4M3 operands (section 2.4), or back to bf16."""
        self._check(lib.engram_set_fp8(self._h, 1 if enable else 0, _stream_ptr(stream)))

    def quantize_e4m3(self, x, q, scale, stream=None):
        """E4M3 codes q (uint8 [rows, cols]) and power-of-two row scales
        (fp32 [rows]) of bf16 x [rows, cols], all on the device."""
        rows, cols = x.shape
        self._check(lib.engram_quantize_e4m3(self._h, _ptr(x), rows, cols, _ptr(q), _ptr(scale),
                                             _stream_ptr(stream)))

    def reserve(self, max_rows: int):
        self._check(lib.engram_reserve(self._h, max_rows))

    def hash(self, tokens, idx, t_begin=0, stream=None):
        B, T = tokens.shape
        self._check(lib.engram_hash(self._h, _ptr(tokens), B, T, t_begin, _ptr(idx),
                                    _stream_ptr(stream)))

    def gather(self, idx, e, stream=None):
        self._check(lib.engram_gather(self._h, _ptr(idx), idx.shape[0], _ptr(e),
                                      _stream_ptr(stream)))

    def forward(self, tokens, h, out, idx=None, t_begin=0, alpha=None, delta=None, stream=None):
        B, T = tokens.shape
        self._check(lib.engram_forward(self._h, _ptr(tokens), _ptr(idx), B, T, t_begin, _ptr(h),
                                       _ptr(out), _ptr(alpha), _ptr(delta), _stream_ptr(stream)))

    def forward_host(self, tokens, h, out, t_begin=0, alpha=None, stream=None):
        """The forward from host tensors (tokens int32 [B, T], h and out [rows, M, d],
        alpha fp32 [rows, M] or None; pinned for overlapped copies): the library
        stages them on the device and copies the result back; `stream` waits for it."""
        for name, t in (("tokens", tokens), ("h", h), ("out", out), ("alpha", alpha)):
            if t is not None and (t.is_cuda or not t.is_contiguous()):
                raise EngramError(ENGRAM_ERR_INVALID, name + " must be a contiguous host tensor")
        B, T = tokens.shape
        rows = B * (T - t_begin)
        M, d = self.cfg.branches, self.cfg.d_hidden
        if tuple(h.shape) != (rows, M, d) or tuple(out.shape) != (rows, M, d):
            raise EngramError(ENGRAM_ERR_INVALID, "h and out must have shape (rows, M, d)")
        if alpha is not None and tuple(alpha.shape) != (rows, M):
            raise EngramError(ENGRAM_ERR_INVALID, "alpha must have shape (rows, M)")
        dt = torch.float32 if self.cfg.dtype == ENGRAM_F32 else torch.bfloat16
        if (tokens.dtype != torch.int32 or h.dtype != dt or out.dtype != dt
                or (alpha is not None and alpha.dtype != torch.float32)):
            raise EngramError(ENGRAM_ERR_INVALID, "dtypes: tokens int32, h and out %s, alpha "
                              "float32" % dt)
        self._check(lib.engram_forward_host(self._h, _ptr(tokens), B, T, t_begin, _ptr(h),
                                            _ptr(out), _ptr(alpha), _stream_ptr(stream)))

    def backward(self, tokens, h, dout, dh, dw_k=None, dw_v=None, dnorm_q=None, dnorm_k=None,
                 dtables=None, idx=None, t_begin=0, stream=None):
        """Gradients of the forward for dL/dout = dout: dh written; dw_k, dw_v,
        dnorm_q, dnorm_k and the S fp32 table gradients accumulated (any may be None)."""
        B, T = tokens.shape
        arr = None
        if dtables is not None:
            # S pointers, or S x N with row-sharded tables
            arr = ctypes.cast((ctypes.c_void_p * len(dtables))(*[t.data_ptr() for t in dtables]),
                              ctypes.c_void_p)
        self._check(lib.engram_backward(self._h, _ptr(tokens), _ptr(idx), B, T, t_begin, _ptr(h),
                                        _ptr(dout), _ptr(dh), _ptr(dw_k), _ptr(dw_v),
                                        _ptr(dnorm_q), _ptr(dnorm_k), arr, _stream_ptr(stream)))

    def backward_host(self, tokens, h, dout, dh, dw_k=None, dw_v=None, dnorm_q=None,
                      dnorm_k=None, dtables=None, t_begin=0, stream=None):
        """The backward from host tensors (tokens, h, dout in; dh out; pinned for
        overlapped copies); the weight and table gradients stay device tensors."""
        for name, t in (("tokens", tokens), ("h", h), ("dout", dout), ("dh", dh)):
            if t.is_cuda or not t.is_contiguous():
                raise EngramError(ENGRAM_ERR_INVALID, name + " must be a contiguous host tensor")
        B, T = tokens.shape
        rows = B * (T - t_begin)
        M, d = self.cfg.branches, self.cfg.d_hidden
        dt = torch.float32 if self.cfg.dtype == ENGRAM_F32 else torch.bfloat16
        for name, t in (("h", h), ("dout", dout), ("dh", dh)):
            if tuple(t.shape) != (rows, M, d) or t.dtype != dt:
                raise EngramError(ENGRAM_ERR_INVALID, "%s must be %s of shape (rows, M, d)" % (name, dt))
        if tokens.dtype != torch.int32:
            raise EngramError(ENGRAM_ERR_INVALID, "tokens must be int32")
        arr = None
        if dtables is not None:
            arr = ctypes.cast((ctypes.c_void_p * len(dtables))(*[t.data_ptr() for t in dtables]),
                              ctypes.c_void_p)
        self._check(lib.engram_backward_host(self._h, _ptr(tokens), B, T, t_begin, _ptr(h),
                                             _ptr(dout), _ptr(dh), _ptr(dw_k), _ptr(dw_v),
                                             _ptr(dnorm_q), _ptr(dnorm_k), arr,
                                             _stream_ptr(stream)))

    def prefetch(self, tokens, t_begin=0, stream=None, want_count=False):
        B, T = tokens.shape
        n = ctypes.c_int64(0)
        self._check(lib.engram_prefetch(self._h, _ptr(tokens), B, T, t_begin, _stream_ptr(stream),
                                        ctypes.byref(n) if want_count else None))
        return n.value if want_count else None

    def prefetch_wait(self):
        """Block until the oldest pending prefetch's rows are in device memory."""
        self._check(lib.engram_prefetch_wait(self._h))

    def set_prefetch(self, mode: str = "host_threads", workers: int = 0):
        """Route of the prefetch's copy from host tables: "host_threads" (host
        threads + copy engines) or "zero_copy" (a kernel of `workers` CTAs);
        workers = 0 takes the route's default."""
        m = {"host_threads": ENGRAM_PREFETCH_HOST_THREADS,
             "zero_copy": ENGRAM_PREFETCH_ZERO_COPY}[mode]
        self._check(lib.engram_set_prefetch(self._h, m, workers))

    def build_hot_cache(self, tokens, max_rows: int, t_begin=0, stream=None):
        """Keep the max_rows rows the calibration tokens address most often in HBM."""
        B, T = tokens.shape
        self._check(lib.engram_build_hot_cache(self._h, _ptr(tokens), B, T, t_begin, max_rows,
                                               _stream_ptr(stream)))

    def prefetch_hot_hits(self) -> int:
        """Distinct rows of the last prefetch served from the hot-row cache."""
        n = ctypes.c_int64(0)
        self._check(lib.engram_prefetch_hot_hits(self._h, ctypes.byref(n)))
        return n.value

    def profile_next_forward(self, events):
        """Record 5 or 6 CUDA events inside the next forward (stage boundaries)."""
        self._prof_keep = list(events)
        n = len(events)
        arr = (ctypes.c_void_p * n)(*[e.cuda_event for e in events])
        self._check(lib.engram_profile_next_forward(self._h, ctypes.cast(arr, ctypes.c_void_p), n))

    def profile_next_backward(self, events):
        """Record 6 CUDA events inside the next backward (stage boundaries)."""
        self._bprof_keep = list(events)
        arr = (ctypes.c_void_p * 6)(*[e.cuda_event for e in events])
        self._check(lib.engram_profile_next_backward(self._h, ctypes.cast(arr, ctypes.c_void_p),
                                                     len(events)))

    def kernel_launches(self) -> int:
        return int(lib.engram_kernel_launches(self._h))

    def project_gate_noalloc(self, e, h, out, alpha=None, stream=None):
        """Projection + gate from caller-supplied memory vectors; allocates nothing.

        e [rows, d_mem], h and out [rows, M, d] in the handle's dtype, alpha
        fp32 [rows, M] or None; all contiguous on the handle's device.  The
        library encodes its tensor maps from these sizes, so they are checked
        here before the call."""
        rows = e.shape[0] if e.dim() == 2 else -1
        dt = torch.float32 if self.cfg.dtype == ENGRAM_F32 else torch.bfloat16
        M, d = self.cfg.branches, self.cfg.d_hidden
        want = [("e", e, (rows, self.d_mem), dt), ("h", h, (rows, M, d), dt),
                ("out", out, (rows, M, d), dt)]
        if alpha is not None:
            want.append(("alpha", alpha, (rows, M), torch.float32))
        for name, t, shape, dtype in want:
            if tuple(t.shape) != shape or t.dtype != dtype or not t.is_contiguous() \
                    or not t.is_cuda:
                raise EngramError(ENGRAM_ERR_INVALID,
                                  "project_gate_noalloc: %s must be a contiguous CUDA tensor of "
                                  "shape %s and dtype %s (got %s %s)"
                                  % (name, shape, dtype, tuple(t.shape), t.dtype))
        self._check(lib.engram_project_gate_noalloc(self._h, _ptr(e), rows, _ptr(h),
                                                    _ptr(out), _ptr(alpha), _stream_ptr(stream)))

    def selftest_timeout(self, stream=None) -> int:
        """Run the bounded-wait expiry self-test; returns ENGRAM_ERR_TIMEOUT if it works."""
        return lib.engram_selftest_timeout(self._h, _stream_ptr(stream))

    def check_errors(self, stream=None) -> int:
        """Synchronise the stream; return the device error status (0 = none)."""
        return lib.engram_check_errors(self._h, _stream_ptr(stream))
