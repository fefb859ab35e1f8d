"""Test helper: one seeded synthetic problem, run through the oracle and the
CUDA path (through the C ABI) on the same inputs.

Only the tests and the smoke check use this module.  The oracle values never
come from the CUDA path: indices are hashed by the oracle from the tokens,
table rows are read at the oracle's own indices.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

import oracle
from hashed_gram_embedding_compress_b200 import synth


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def to_oracle(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return bf16_bits(t)
    return t.detach().contiguous().cpu().numpy()


def from_bits(a: np.ndarray, dtype: str) -> torch.Tensor:
    if dtype == "bf16":
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16)
    return torch.from_numpy(a.copy())


def rel_l2(x, y) -> float:
    x = torch.as_tensor(x).double()
    y = torch.as_tensor(y).double()
    den = torch.linalg.vector_norm(y).item()
    return torch.linalg.vector_norm(x - y).item() / max(den, 1e-300)


@dataclass
class Problem:
    shape: synth.EngramShape
    device: str = "cuda"
    seeds: dict = field(default_factory=dict)

    def __post_init__(self):
        sh = self.shape
        self.seeds = synth.stream_seeds(sh)
        self.tokens = synth.make_tokens(sh, self.seeds)
        self.comp_map = synth.make_comp_map(sh, self.seeds)
        self.hash_seed = synth.make_hash_seed(self.seeds)
        # the oracle's own indices and table sizes
        self.c, self.z, self.mult, self.primes = oracle.forward_indices(
            self.tokens.numpy(), self.comp_map.numpy(), sh.cvocab, sh.orders, sh.heads,
            self.hash_seed, sh.rows_target, t_begin=sh.t_begin)
        pin = sh.table_location == "pinned_host"
        self.tables = synth.make_tables([int(p) for p in self.primes], sh.d_head, sh.dtype,
                                        self.seeds, device=self.device, pin=pin)
        w_k, w_v, nq, nk = synth.make_weights(sh, self.seeds)
        self.w_k_cpu, self.w_v_cpu, self.nq_cpu, self.nk_cpu = w_k, w_v, nq, nk
        self.w_k, self.w_v = w_k.to(self.device), w_v.to(self.device)
        self.norm_q, self.norm_k = nq.to(self.device), nk.to(self.device)
        self.h = synth.make_hidden(sh, self.seeds, device=self.device)

    # ------------------------------------------------------------ CUDA path
    def engram(self, eps: float = 1e-6, flags: int = 0):
        from hashed_gram_embedding_compress_b200 import engram as eg
        sh = self.shape
        cfg = eg.make_config(vocab=sh.vocab, cvocab=sh.cvocab, comp_map=self.comp_map,
                             orders=sh.orders, heads=sh.heads, d_head=sh.d_head,
                             d_hidden=sh.d_hidden, branches=sh.branches, dtype=sh.dtype, eps=eps,
                             table_rows_target=sh.rows_target, hash_seed=self.hash_seed,
                             table_location=sh.table_location, flags=flags)
        m = eg.Engram(cfg)
        m.set_params(self.tables, self.w_k, self.w_v, self.norm_q, self.norm_k)
        return m

    # --------------------------------------------------------------- oracle
    def table_rows(self, rows: np.ndarray):
        """Per-table arrays holding only the rows the oracle addresses for `rows`,
        and the indices into them (the oracle gathers from these)."""
        z = self.z[rows]
        mini, zz = [], np.empty_like(z)
        for s, t in enumerate(self.tables):
            idx = torch.from_numpy(z[:, s]).to(t.device)
            mini.append(to_oracle(t[idx]))
            zz[:, s] = np.arange(len(rows))
        return mini, zz

    def oracle_forward(self, rows: np.ndarray, eps: float = 1e-6, fp8: bool = False):
        """e, alpha, delta, out at `rows`; fp8: the projections on E4M3 operands
        (section 2.4), e quantised per row and W per output channel."""
        mini, zz = self.table_rows(rows)
        e = oracle.gather(mini, zz)
        h = to_oracle(self.h[torch.from_numpy(rows).to(self.h.device)])
        args = (e, to_oracle(self.w_k_cpu), to_oracle(self.w_v_cpu), self.nq_cpu.numpy(),
                self.nk_cpu.numpy(), h, eps)
        if fp8:
            if getattr(self, "_w8", None) is None:
                self._w8 = oracle.quantize_weights_e4m3(args[1], args[2])
            alpha, delta, out = oracle.project_gate_fp8(*args, weights=self._w8)
        else:
            alpha, delta, out = oracle.project_gate(*args)
        return e, alpha, delta, out

    def conv_weights(self, kernel_size: int = 4):
        """Seeded ShortConv weights (conv_w [d, W], norm_w [d], fp32 on the CPU)."""
        return synth.make_conv_weights(self.shape, self.seeds, kernel_size)

    def oracle_forward_conv(self, rows: np.ndarray, conv_w, norm_w, dilation: int,
                            eps: float = 1e-6, fp8: bool = False):
        """Y [n, M, d] (double) and out [n, M, d] (h's dtype) of Eq. (5) at `rows`
        (t_begin = 0, row = b T + t): the gated values alpha v are formed by
        the oracle at the positions the taps read, t - i * dilation."""
        sh = self.shape
        assert sh.t_begin == 0
        W = conv_w.shape[1]
        T = sh.T
        need = sorted({int(r) - i * dilation for r in rows for i in range(W)
                       if (int(r) % T) - i * dilation >= 0})
        need = np.array(need, dtype=np.int64)
        _, _, vt, _ = self.oracle_forward(need, eps, fp8)     # delta = alpha v [n, M, d]
        pos = {int(r): j for j, r in enumerate(need)}
        M, d = sh.branches, sh.d_hidden
        cw, nw = conv_w.numpy(), norm_w.numpy()
        Y = np.empty((len(rows), M, d))
        for j, r in enumerate(rows):
            r = int(r)
            have = np.array([(r % T) - i * dilation >= 0 for i in range(W)], dtype=np.int32)
            for m in range(M):
                taps = np.zeros((W, d))
                for i in range(W):
                    if have[i]:
                        taps[i] = vt[pos[r - i * dilation], m]
                Y[j, m] = oracle.short_conv_at(taps, have, cw, nw, eps)
        h = to_oracle(self.h[torch.from_numpy(np.asarray(rows)).to(self.h.device)])
        out = oracle.add_round(h, Y.reshape(h.shape))
        return Y, out

    def sample_rows(self, n: int, seed: int = 0) -> np.ndarray:
        """Every sequence's first three and last emitted positions, plus random rows."""
        sh = self.shape
        Tout = sh.T - sh.t_begin
        must = []
        for b in range(sh.B):
            for t in (0, 1, 2, Tout - 1):
                if 0 <= t < Tout:
                    must.append(b * Tout + t)
        must = np.unique(np.array(must, dtype=np.int64))
        rng = np.random.default_rng(seed)
        extra = rng.choice(sh.rows_out, size=min(n, sh.rows_out), replace=False)
        return np.unique(np.concatenate([must, extra]))


def out_close(out_gpu: np.ndarray, out_ref: np.ndarray, dtype: str, h: Optional[np.ndarray] = None):
    """Comparison of `out` (h's dtype) against the oracle's rounded out."""
    if dtype == "f32":
        return float(np.abs(out_gpu.astype(np.float64) - out_ref.astype(np.float64)).max())
    g = from_bits(out_gpu, "bf16").double()
    r = from_bits(out_ref, "bf16").double()
    return rel_l2(g, r)
