"""Seeded synthetic inputs for the Engram lookup-and-gate forward.

This module draws random inputs only.  It holds none of the method's
arithmetic (no compression, hashing, gathering, projection or gating), so both
the CUDA path and the CPU oracle may consume what it produces.

The pages' real workloads (the 128k tokenizer, its NFKC/lower-case merge map,
the training corpus and trained weights) are not available.  These stand in:

* tokens: Zipf by rank, P(r) ~ r^-s over r = 1..V, drawn by inverse-CDF in
  double precision and sent to ids through a seeded permutation (natural
  n-grams are Zipfian: "Conditional Memory via Scalable Lookup", section 2.5);
* compression map: a seeded surjection V -> V'.  V' raw ids are sent onto a
  permutation of [0, V'); the other V - V' ids go to targets drawn from a
  Zipf(1.0) over [0, V'), so merge groups are heavy-tailed (the same paper,
  Appendix C, Table 6 lists groups of 163, 54, 40, 35 and 30 raw ids);
* hash seed: one uint64 per problem (the multipliers are derived from it by
  each side from the published SplitMix64 definition);
* tables: N(0, 0.02^2) rows;  W_K, W_V: N(0, 1/fan_in) with fan_in = d_mem;
  hidden states: N(0, 1);  RMSNorm weights: 1 + 0.1 N(0, 1).

Small tensors are drawn on the CPU with a seeded ``torch.Generator``; tables
and hidden states may be drawn on a CUDA device with a seeded CUDA generator
(their values then differ from a CPU draw, but every consumer reads the same
tensor).
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np
import torch

BASE_SEED = 20261202

#: names of the independent sub-streams of one problem
# appended streams keep the seeds of the earlier ones (SeedSequence children by index)
STREAMS = ("tokens", "map", "hash", "tables", "weights", "hidden", "norms", "conv", "dout")


@dataclass(frozen=True)
class EngramShape:
    """Sizes of one synthetic problem (names follow the paper's notation)."""

    name: str
    index: int                 # seed offset
    vocab: int                 # V
    cvocab: int                # V'
    zipf_s: float              # token Zipf exponent
    B: int                     # sequences
    T: int                     # tokens per sequence
    t_begin: int               # first position that is emitted (decode: T-1)
    orders: tuple              # n-gram orders, ascending
    heads: int                 # K hash heads per order
    rows_target: int           # table rows: primes >= this value
    d_head: int                # d_h: columns of one table
    d_hidden: int              # d
    branches: int              # M
    dtype: str                 # "f32" or "bf16" (tables, weights, hidden)
    table_location: str = "device"   # "device" or "pinned_host"

    @property
    def num_tables(self) -> int:
        return len(self.orders) * self.heads

    @property
    def d_mem(self) -> int:
        return self.num_tables * self.d_head

    @property
    def rows_out(self) -> int:
        return self.B * (self.T - self.t_begin)

    def replace(self, **kw) -> "EngramShape":
        return dataclasses.replace(self, **kw)


SHAPES = {
    "tiny_f32": EngramShape("tiny_f32", 1, 1000, 770, 1.1, 2, 64, 0, (2, 3), 4,
                            10007, 32, 128, 1, "f32"),
    "prefill_bf16": EngramShape("prefill_bf16", 2, 32768, 25231, 1.1, 8, 4096, 0,
                                (2, 3), 8, 1 << 20, 80, 2560, 1, "bf16"),
    "decode_mb": EngramShape("decode_mb", 3, 32768, 25231, 1.1, 256, 3, 2, (2, 3), 8,
                             1 << 20, 80, 2560, 4, "bf16"),
    "large_hbm": EngramShape("large_hbm", 4, 128000, 98560, 1.05, 4, 8192, 0, (2, 3), 8,
                             1 << 24, 80, 4096, 4, "bf16"),
    "offload": EngramShape("offload", 5, 128000, 98560, 1.05, 4, 8192, 0, (2, 3), 8,
                           1 << 24, 80, 4096, 4, "bf16", "pinned_host"),
}


def torch_dtype(dtype: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[dtype]


def stream_seeds(shape: EngramShape, extra: int = 0) -> dict:
    """One integer seed per sub-stream, from SeedSequence.spawn."""
    ss = np.random.SeedSequence([BASE_SEED + shape.index, extra])
    kids = ss.spawn(len(STREAMS))
    return {n: int(k.generate_state(1, dtype=np.uint64)[0] & 0x7FFFFFFFFFFFFFFF)
            for n, k in zip(STREAMS, kids)}


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def zipf_ids(n: int, vocab: int, s: float, g: torch.Generator) -> torch.Tensor:
    """n draws of Zipf(s) ranks over 1..vocab, sent to ids by a permutation."""
    r = torch.arange(1, vocab + 1, dtype=torch.float64)
    p = r.pow(-s)
    cdf = torch.cumsum(p, 0)
    cdf = cdf / cdf[-1]
    u = torch.rand(n, generator=g, dtype=torch.float64)
    rank = torch.searchsorted(cdf, u).clamp_(max=vocab - 1)
    perm = torch.randperm(vocab, generator=g)
    return perm[rank].to(torch.int32)


def make_tokens(shape: EngramShape, seeds: dict) -> torch.Tensor:
    """int32 [B, T] raw token ids in [0, V)."""
    g = _gen(seeds["tokens"])
    return zipf_ids(shape.B * shape.T, shape.vocab, shape.zipf_s, g).view(shape.B, shape.T)


def make_comp_map(shape: EngramShape, seeds: dict) -> torch.Tensor:
    """int32 [V]: a seeded surjection of [0, V) onto [0, V')."""
    V, Vc = shape.vocab, shape.cvocab
    assert 0 < Vc <= V
    g = _gen(seeds["map"])
    raw = torch.randperm(V, generator=g)
    out = torch.empty(V, dtype=torch.int32)
    out[raw[:Vc]] = torch.randperm(Vc, generator=g).to(torch.int32)
    if V > Vc:
        out[raw[Vc:]] = zipf_ids(V - Vc, Vc, 1.0, g)
    return out


def make_hash_seed(seeds: dict) -> int:
    return int(np.random.SeedSequence(seeds["hash"]).generate_state(1, dtype=np.uint64)[0])


def make_tables(rows: Sequence[int], d_head: int, dtype: str, seeds: dict,
                device="cpu", chunk_elems: int = 1 << 26, pin: bool = False):
    """One [rows[s], d_head] tensor per table, N(0, 0.02^2), on `device`.

    With ``pin`` the tables are drawn on `device` and copied into pinned host
    memory (page-locked, so a kernel can read them over PCIe).
    """
    dt = torch_dtype(dtype)
    g = _gen(seeds["tables"], device)
    out = []
    for r in rows:
        dst_dev = "cpu" if pin else device
        t = torch.empty((int(r), d_head), dtype=dt, device=dst_dev, pin_memory=pin)
        step = max(1, chunk_elems // d_head)
        for a in range(0, int(r), step):
            b = min(int(r), a + step)
            x = torch.randn((b - a, d_head), generator=g, device=device, dtype=torch.float32)
            x.mul_(0.02)
            t[a:b].copy_(x.to(dt))
        out.append(t)
    return out


def make_weights(shape: EngramShape, seeds: dict):
    """W_K [M, d, d_mem], W_V [d, d_mem] (shape.dtype), norm_q, norm_k fp32 [M, d]."""
    dt = torch_dtype(shape.dtype)
    M, d, dm = shape.branches, shape.d_hidden, shape.d_mem
    g = _gen(seeds["weights"])
    std = 1.0 / np.sqrt(dm)
    w_k = (torch.randn((M, d, dm), generator=g) * std).to(dt)
    w_v = (torch.randn((d, dm), generator=g) * std).to(dt)
    gn = _gen(seeds["norms"])
    norm_q = 1.0 + 0.1 * torch.randn((M, d), generator=gn)
    norm_k = 1.0 + 0.1 * torch.randn((M, d), generator=gn)
    return w_k, w_v, norm_q.float(), norm_k.float()


def make_conv_weights(shape: EngramShape, seeds: dict, kernel_size: int = 4):
    """ShortConv weights (Eq. 5): conv_w [d, W] (tap i multiplies position
    t - i * dilation) with N(0, 0.5^2) entries, so the conv output is O(1) and
    SiLU is exercised on both sides of zero (the paper initialises them to
    zero, which makes the conv the identity); norm_w [d] = 1 + 0.1 N(0, 1).
    Both fp32."""
    g = _gen(seeds["conv"])
    d = shape.d_hidden
    conv_w = 0.5 * torch.randn((d, kernel_size), generator=g)
    norm_w = 1.0 + 0.1 * torch.randn((d,), generator=g)
    return conv_w.float(), norm_w.float()


def make_hidden(shape: EngramShape, seeds: dict, device="cpu", rows: Optional[int] = None,
                chunk_elems: int = 1 << 26, stream: str = "hidden") -> torch.Tensor:
    """h [rows_out, M, d] ~ N(0, 1) in shape.dtype."""
    dt = torch_dtype(shape.dtype)
    n = shape.rows_out if rows is None else rows
    per = shape.branches * shape.d_hidden
    g = _gen(seeds[stream], device)
    h = torch.empty((n, shape.branches, shape.d_hidden), dtype=dt, device=device)
    step = max(1, chunk_elems // per)
    for a in range(0, n, step):
        b = min(n, a + step)
        h[a:b].copy_(torch.randn((b - a, shape.branches, shape.d_hidden), generator=g,
                                 device=device, dtype=torch.float32).to(dt))
    return h


def make_grad_out(shape: EngramShape, seeds: dict, device="cpu") -> torch.Tensor:
    """dL/dout [rows_out, M, d] ~ N(0, 1) in shape.dtype, for the backward."""
    return make_hidden(shape, seeds, device=device, stream="dout")
