"""Throughput of the Engram forward (hash + gather + projections + gate) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one engram_forward over one batch of the prefill workload
(B=8 sequences x T=4096 tokens, 16 tables of ~2^20 rows x 80 bf16, d=2560,
M=1): compress, hash, gather, key and value projections, gate, residual.
`value` is tokens/s with every input resident in HBM; `e2e` is the same call
with the inputs in pinned host memory, copied in and the output copied out
inside the timed region.  Inputs are larger than L2 (h 168 MB in, 168 MB out,
tables 2.7 GB), so no L2 flush runs between steps.

With N > 1 (torchrun), every rank runs its own replica on its own seeded batch
(the forward has no cross-rank exchange); the time is the max over ranks.

--impl reference times the CPU oracle (plain single-threaded C, fp64) on a
bounded sample of the same workload: the reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Engram fwd tokens/s (hash+gather+gate); gather GB/s as % of HBM peak"
WORKLOAD = "prefill_bf16"
DESCRIBE = {
    "prefill_bf16": "prefill_bf16: B=8 x T=4096 tokens, vocab 32768->25231, orders {2,3} x 8 heads, "
                    "16 tables of primes >= 2^20 rows x 80 bf16 (d_mem 1280), d=2560, M=1, "
                    "fp32 accumulate",
    "decode_mb": "decode_mb: B=256 sequences, 1 new token each after a 2-token prefix, tables as "
                 "prefill_bf16, M=4 branches (own W_K 1280->2560 and RMSNorm weights each, shared "
                 "W_V), h [256,4,2560] bf16",
    "large_hbm": "large_hbm: B=4 x T=8192 tokens, vocab 128000->98560, 16 tables of primes >= 2^24 "
                 "rows x 80 bf16 (43 GB in HBM), d=4096, M=4",
    "offload": "offload: large_hbm shapes with the tables in pinned host memory, rows prefetched "
               "over PCIe one step ahead on a side stream, overlapped with a 4096^3 bf16 GEMM "
               "standing in for the preceding backbone block",
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=None,
                    help="steps of the end-to-end (host-buffer) measurement; default: enough "
                         "for ~0.1 s, at least 10, from one untimed step's wall time")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="budget of the oracle's timed sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default="prefill_bf16",
                    choices=["prefill_bf16", "decode_mb", "large_hbm", "offload"],
                    help="prefill_bf16 is the benchmarked line; the others measure the other "
                         "configurations of the same forward")
    ap.add_argument("--short-conv", action="store_true",
                    help="with the short convolution of Eq. 5 (W = 4, dilation = the largest "
                         "n-gram order, seeded non-zero weights); prefill-type workloads")
    ap.add_argument("--fp8", action="store_true",
                    help="projections on E4M3 operands (section 2.4's FP8 matmul): e quantised "
                         "per row inside the gather, W per output channel; prefill-type workloads")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward (training) step instead of the forward: gradients "
                         "of h, W_K, W_V, the RMSNorm weights and the tables for a seeded dL/dout")
    ap.add_argument("--graph", action="store_true",
                    help="replay each step from a captured CUDA graph (launch-bound shapes)")
    ap.add_argument("--graph-steps", type=int, default=None,
                    help="with --graph: consecutive steps captured in one graph (the launches of "
                         "one step then overlap the next step's, as in eager calls); --steps "
                         "must be a multiple of it (default: the largest of 8, 4, 2, 1 that "
                         "divides --steps)")
    ap.add_argument("--offload-gb", type=float, default=100.0,
                    help="offload workload: total size of the pinned host tables")
    ap.add_argument("--hot-rows", type=int, default=0,
                    help="offload workload: rows of the HBM hot-row cache in front of the host "
                         "tables, chosen from 4 calibration batches of other tokens (0: none)")
    ap.add_argument("--load-seconds", type=float, default=1.5,
                    help="back-to-back steps before the timed ones, so that the clock sampler "
                         "sees the loaded state (0 for profiling captures)")
    ap.add_argument("--rows-target", type=int, default=None,
                    help="smaller tables for profiling captures (same kernel shapes); "
                         "not the benchmarked workload")
    return ap.parse_args()


def load_peaks():
    """HBM GB/s and the dense bf16 TFLOP/s of this GPU: (hbm, burst, sustained, source).

    The projection launches last 0.1-1 ms inside a timed region of tens of
    milliseconds, not a seconds-long loop, so the burst GEMM figure is their
    denominator; the sustained one (cuBLAS back to back for seconds under the
    power cap) is reported beside it."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return (d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "measured")
    return 6650.0, 1590.0, 1400.0, "fallback"


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.lines = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0=None, t1=None):
        """Median SM clock and active throttle reasons of samples in [t0, t1]."""
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, ln in self.lines:
            if (t0 is not None and ts < t0) or (t1 is not None and ts > t1):
                continue
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------ the workload

def draw_inputs(rank: int, device, primes, rows_target=None, workload=WORKLOAD, short_conv=False):
    """The seeded synthetic inputs of one rank's batch (no library call): tokens,
    map, tables of the given prime sizes, weights, hidden states, conv weights."""
    from hashed_gram_embedding_compress_b200 import synth

    sh = synth.SHAPES[workload]
    if rows_target:
        sh = sh.replace(rows_target=rows_target)
    seeds = rank_seeds(rank, workload)
    tokens = synth.make_tokens(sh, seeds)
    comp_map = synth.make_comp_map(sh, seeds)
    tables = synth.make_tables([int(p) for p in primes], sh.d_head, sh.dtype, seeds, device=device)
    w_k, w_v, nq, nk = synth.make_weights(sh, seeds)
    w_k, w_v, nq, nk = w_k.to(device), w_v.to(device), nq.to(device), nk.to(device)
    h = synth.make_hidden(sh, seeds, device=device)
    conv = None
    if short_conv:
        cw, nw = synth.make_conv_weights(sh, seeds, 4)
        conv = (cw.to(device), nw.to(device), 4, max(sh.orders))
    return dict(sh=sh, tokens=tokens, comp_map=comp_map, tables=tables, w_k=w_k, w_v=w_v,
                nq=nq, nk=nk, h=h, seeds=seeds, hash_seed=synth.make_hash_seed(seeds),
                primes=primes, conv=conv)


def setup(rank: int, device, rows_target=None, workload=WORKLOAD, short_conv=False, fp8=False):
    """One rank's handle of the library with its parameters set, and its inputs."""
    from hashed_gram_embedding_compress_b200 import engram as eg
    from hashed_gram_embedding_compress_b200 import synth

    sh = synth.SHAPES[workload]
    if rows_target:
        sh = sh.replace(rows_target=rows_target)
    seeds = rank_seeds(rank, workload)
    cfg = eg.make_config(vocab=sh.vocab, cvocab=sh.cvocab,
                         comp_map=synth.make_comp_map(sh, seeds), orders=sh.orders,
                         heads=sh.heads, d_head=sh.d_head, d_hidden=sh.d_hidden,
                         branches=sh.branches, dtype=sh.dtype, eps=1e-6,
                         table_rows_target=sh.rows_target, hash_seed=synth.make_hash_seed(seeds))
    m = eg.Engram(cfg)
    primes, _ = m.hash_params()
    P = draw_inputs(rank, device, primes, rows_target, workload, short_conv)
    m.set_params(P["tables"], P["w_k"], P["w_v"], P["nq"], P["nk"])
    if P["conv"] is not None:
        m.set_short_conv(*P["conv"])
    if fp8:
        m.set_fp8(True)
    m.reserve(sh.rows_out)
    return P | dict(m=m, fp8=fp8)


def algorithmic(sh, fp8=False):
    """Per-step algorithmic work: bytes of the gather and hash, FLOPs and bytes of the projections.
    fp8: e is written as one E4M3 byte per element plus a 4-byte scale per row."""
    R, S, dm, d, M = sh.rows_out, sh.num_tables, sh.d_mem, sh.d_hidden, sh.branches
    elt = 2 if sh.dtype == "bf16" else 4
    row_bytes = sh.d_head * elt
    if sh.table_location == "device":
        # hash fused into the gather: tokens read, table rows read, e written
        gather_bytes = R * S * row_bytes * 2 + sh.B * sh.T * 4
        if fp8:
            gather_bytes = R * S * row_bytes + R * (dm + 4) + sh.B * sh.T * 4
        hash_bytes = 0
    else:
        gather_bytes = R * S * (row_bytes * 2 + 8)   # rows read, e written, indices read
        hash_bytes = R * S * 8 + sh.B * sh.T * 4     # indices written, tokens read
    gemm_flops = 2.0 * R * dm * (M * d + d)          # [W_K^(1..M); W_V] e
    # key kernel: e read, W_K read, h read; value kernel: e, W_V, h read, out written
    op = 1 if fp8 else elt                           # bytes per operand element of the matmul
    gemm_bytes = (2 * R * dm * op + (M * d + d) * dm * op + 3 * R * M * d * elt)
    # short conv: v (fp32) read once, h read and out written per branch, plus
    # alpha and the per-tile sums of v^2
    conv_bytes = R * d * 4 + 2 * R * M * d * elt + R * (M + d // 256) * 4
    # the whole step's unavoidable traffic: tokens in, each addressed table row
    # read once, h read once and out written once, the weights read once (e,
    # k and v need never reach HBM)
    step_bytes = (sh.B * sh.T * 4 + R * S * row_bytes + 2 * R * M * d * elt
                  + (M * d + d) * dm * op)
    return dict(gather_bytes=gather_bytes, hash_bytes=hash_bytes, gemm_flops=gemm_flops,
                conv_bytes=conv_bytes, step_bytes=step_bytes,
                gemm_bytes=gemm_bytes)


def step_roofline(A, ms_step, hbm_gbs, tflops):
    """The whole step against its roofline: the slower of its unavoidable HBM
    bytes at the measured copy bandwidth and its GEMM FLOPs at the tensor peak."""
    t_mem = A["step_bytes"] / (hbm_gbs * 1e9) * 1e3
    t_mma = A["gemm_flops"] / (tflops * 1e12) * 1e3
    t = max(t_mem, t_mma)
    return {"bound": "tensor" if t_mma >= t_mem else "hbm", "time_ms": t,
            "bytes": A["step_bytes"], "flops": A["gemm_flops"], "frac": t / ms_step,
            "peak_tflops": tflops, "peak_gbs": hbm_gbs}


def kernel_traffic(name="traffic.json", key="proj_gate_bytes_per_step"):
    """DRAM bytes from a committed ncu capture (by default those of the
    projection kernel's key + value launches per step), or None once the
    captured kernel's source has changed."""
    p = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    h = hashlib.sha256()
    for f in d.get("sources", []):
        h.update(open(os.path.join(ROOT, f), "rb").read())
    if d.get("source_sha256_16") != h.hexdigest()[:16]:
        return None
    return d.get(key)


def e2e_count(requested, step, dist, target_s=0.1, lo=10, hi=2000) -> int:
    """Steps of an end-to-end measurement: as requested, else enough for about
    target_s of work (at least lo), from one more untimed step's wall time; the
    largest over ranks, so that every rank takes the same steps."""
    import torch
    if requested:
        return max(1, requested)
    t = time.monotonic()
    step()
    torch.cuda.synchronize()
    n = int(min(hi, max(lo, target_s / max(time.monotonic() - t, 1e-6))))
    if dist:
        v = torch.tensor([n], device="cuda", dtype=torch.int64)
        dist.all_reduce(v, op=dist.ReduceOp.MAX)
        n = int(v.item())
    return n


def max_over_ranks(x: float, dist, device) -> float:
    """The largest value of x over all ranks (identity without a process group)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seeds(rank: int, workload: str = WORKLOAD):
    """Each rank draws its own batch: independent replicas (weak scaling)."""
    from hashed_gram_embedding_compress_b200 import synth
    return synth.stream_seeds(synth.SHAPES[workload], extra=rank)


def run_ours(args, rank, world, dist):
    import torch

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    P = setup(rank, device, args.rows_target, args.workload, args.short_conv, args.fp8)
    sh, m = P["sh"], P["m"]
    NEV = 6 if args.short_conv else 5  # stage events per forward
    tok_d = P["tokens"].to(device)
    h = P["h"]
    stream = torch.cuda.current_stream()

    # the residual update H <- H + Y in place: out aliases h
    def forward_once():
        m.forward(tok_d, h, h, t_begin=sh.t_begin, stream=torch.cuda.current_stream())

    graph = None
    G = 1
    if args.graph:
        G = (max(1, args.graph_steps) if args.graph_steps
             else next(g for g in (8, 4, 2, 1) if args.steps % g == 0))
    if args.graph:
        if args.steps % G:
            raise SystemExit("--steps must be a multiple of --graph-steps")
        forward_once()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        n0 = m.kernel_launches()
        with torch.cuda.graph(graph):
            for _ in range(G):
                forward_once()
        per_replay = m.kernel_launches() - n0  # kernels each replay launches
        torch.cuda.synchronize()

    def step():
        # one replay covers G steps (G = 1 without a graph)
        if graph is not None:
            graph.replay()
        else:
            forward_once()

    clk = ClockSampler(local).__enter__()
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if m.check_errors(stream) != 0:
        raise RuntimeError("device error during warm-up")
    # keep the GPU under the same back-to-back load for >= 1.5 s before the
    # timed steps, so that the clock sampler sees the loaded state
    t_load = time.monotonic()
    while time.monotonic() - t_load < args.load_seconds:
        for _ in range(50):
            step()
        torch.cuda.synchronize()

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(NEV)] for _ in range(K)]
    for row in evs:  # torch creates the CUDA event at its first record
        for ev in row:
            ev.record(stream)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = m.kernel_launches()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    # the timed steps carry no stage events: an event between two launches
    # would serialise the launches that otherwise overlap (the key launch
    # starts during the gather, the value launch during the key launch)
    t0.record(stream)
    for k in range(K // G):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    t_end = time.monotonic()
    launches = m.kernel_launches() - launches0
    if graph is not None:
        launches = per_replay * (K // G)  # replays do not pass through the library's counter
    # stage times: the same steps again, each with events between its launches
    if graph is None:
        for k in range(K):
            m.profile_next_forward(evs[k])
            step()
        torch.cuda.synchronize()
    time.sleep(0.3)
    clk.__exit__(None, None, None)
    if dist:
        dist.barrier()
    ms = max_over_ranks(t0.elapsed_time(t1), dist, device)
    if graph is None:
        stage = [[evs[k][i].elapsed_time(evs[k][i + 1]) for i in range(NEV - 1)] for k in range(K)]
        # hash, gather, key, value (, short conv)
        st_mean = [sum(s[i] for s in stage) / K for i in range(NEV - 1)]
    else:
        # one graph replay per step: no per-kernel events; split by the same
        # shares would be a guess, so the stages are timed by replaying the
        # eager forward once more with events
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(NEV)]
        for e_ in ev:
            e_.record(stream)
        st_mean = [0.0] * (NEV - 1)
        for _ in range(5):
            m.profile_next_forward(ev)
            forward_once()
            torch.cuda.synchronize()
            for i in range(NEV - 1):
                st_mean[i] += ev[i].elapsed_time(ev[i + 1]) / 5
    if m.check_errors(stream) != 0:
        raise RuntimeError("device error during the timed steps")

    # ------------------------------------------------------------- e2e
    # through the host-buffer entry point: every step copies its tokens and h
    # from pinned host memory to the device and its out back (the library
    # overlaps one step's copies in with the previous step's copies out)
    tok_h = P["tokens"].pin_memory()
    h_h = h.cpu().pin_memory()
    out_h = torch.empty_like(h_h).pin_memory()

    def e2e_step():
        m.forward_host(tok_h, h_h, out_h, t_begin=sh.t_begin, stream=stream)

    e2e_step()
    torch.cuda.synchronize()
    E = e2e_count(args.e2e_steps, e2e_step, dist)
    if dist:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(E):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, device)
    if dist:
        dist.barrier()
    if rank != 0:
        return None

    hbm, tflops_burst, tflops_sus, peak_kind = load_peaks()
    A = algorithmic(sh, args.fp8)
    if args.fp8:
        # E4M3 operands: the nominal dense FP8 rate is twice the bf16 one (4.5 vs 2.25
        # PFLOP/s), applied to the measured bf16 figures
        tflops_burst, tflops_sus = 2 * tflops_burst, 2 * tflops_sus
    tokens_per_step = sh.rows_out
    value = tokens_per_step * world * K / (ms / 1e3)
    gemm_s = (st_mean[2] + st_mean[3]) / 1e3
    gemm_tflops = A["gemm_flops"] / gemm_s / 1e12
    fused = sh.table_location == "device"  # one hash + gather kernel: its time is stage 1
    # calls of at most 256 rows: keys, alpha and values in one launch (stage 2)
    short_fused = (sh.rows_out <= 256 and sh.dtype == "bf16" and sh.d_hidden % 256 == 0
                   and sh.branches <= 4 and not args.fp8 and not args.short_conv)
    gather_s = (st_mean[0] + st_mean[1] if fused else st_mean[1]) / 1e3
    gather_gbs = A["gather_bytes"] / gather_s / 1e9
    # the DRAM bytes the fused kernel moves in the step (row over-fetch and the
    # write-back of the value launch's dirty h included), from an ncu capture
    gather_traffic = (kernel_traffic("traffic_gather.json", "dram_bytes_per_launch")
                      if fused and not args.fp8 and args.workload == WORKLOAD else None)
    traffic = None if args.fp8 else kernel_traffic()
    res = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": max(3, args.warmup),
        "ms_per_step": ms / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3" if args.fp8 else "bf16",
        "data": "synthetic",
        "config": {
            "workload": DESCRIBE[args.workload],
            "global_batch": tokens_per_step * world,
            "seq_len": sh.T,
            "parallelism": "replicas" if world > 1 else "single",
            "l2": "no flush: inputs larger than L2 (h %.0f MB read and written, tables %.1f GB)"
                  % (h.numel() * h.element_size() / 1e6,
                     sum(t.numel() * t.element_size() for t in P["tables"]) / 1e9),
            "residual": "in place: out aliases h (H <- H + alpha v)",
            "cuda_graph": bool(graph is not None),
            "graph_steps": G if graph is not None else None,
        },
        "roofline": {
            "kernel": ("proj_gate_fused_kernel: keys, alpha and values in one launch (256 x 256 "
                       "key and 256 x 128 value CTA-pair tiles, tcgen05)" if short_fused else
                       "proj_gate_pair_kernel (keys, 256 x 256 CTA-pair tiles) + row_alpha_kernel "
                       "+ proj_gate_kernel (values, 128 x 64 single-CTA tiles), tcgen05"
                       if sh.rows_out <= 4096 else
                       "proj_gate_wide_kernel: key + in-place value launches per step (tcgen05, "
                       "CTA pairs)"),
            "bound": "tensor",
            "achieved": gemm_tflops,
            "peak": tflops_burst,
            "unit": "TFLOP/s",
            "frac": gemm_tflops / tflops_burst,
            "traffic": traffic,
            "peak_source": "%s bf16 burst (cuBLAS, best of 10)%s: the launches are 0.1-1 ms "
                           "inside a timed region of tens of ms" % (
                               peak_kind, " x 2, the nominal FP8 / bf16 ratio" if args.fp8 else ""),
            "peak_sustained": tflops_sus,
            "frac_of_sustained": gemm_tflops / tflops_sus,
        },
        "step_roofline": step_roofline(A, ms / K, hbm, tflops_burst),
        "gather": {
            "kernel": ("hash_gather_e4m3_kernel" if args.fp8 else "hash_gather_kernel")
                      if fused else "gather_kernel",
            "achieved_gbs": gather_gbs,
            "frac_of_hbm": gather_gbs / hbm,
            "peak_gbs": hbm,
            "bytes_per_step": A["gather_bytes"],
            "traffic": gather_traffic,
            "traffic_frac_of_hbm": (gather_traffic / gather_s / 1e9 / hbm
                                    if gather_traffic else None),
        },
        "stages_ms": ({"hash_gather": st_mean[0] + st_mean[1]} if fused else
                      {"hash": st_mean[0], "gather": st_mean[1]}) |
                     ({"proj_gate": st_mean[2] + st_mean[3]} if short_fused else
                      {"key_proj_gate": st_mean[2], "value_proj_gate": st_mean[3]}) |
                     ({"short_conv": st_mean[4]} if args.short_conv else {}),
        "e2e": {
            "value": tokens_per_step * world * E / (e2e_ms / 1e3),
            "unit": "tokens/s",
            "h2d_bytes_per_step": tok_h.numel() * 4 + h_h.numel() * h_h.element_size(),
            "d2h_bytes_per_step": out_h.numel() * out_h.element_size(),
            "steps": E,
            "path": "engram_forward_host: C ABI call on pinned host buffers (tokens, h in; out "
                    "back), copies inside the timed region",
        },
        "gpu_launches": launches,
        "clocks": dict(clk.summary(t_load + 0.5, t_end + 0.15),
                       window="last 1 s of back-to-back warm-up steps and the timed steps"),
        "stages_note": "stage times from a second pass of the same steps with events between "
                       "the launches (which serialises them); ms_per_step has no events",
    }
    if args.short_conv:
        res["config"]["workload"] += (" + ShortConv (Eq. 5: W=4, dilation %d, RMSNorm, SiLU, "
                                      "seeded non-zero weights)" % max(sh.orders))
        res["config"]["residual"] = "in place: out aliases h (H <- H + Y, Eq. 5)"
        res["short_conv"] = {
            "kernel": "short_conv_kernel",
            "bound": "hbm",
            "achieved_gbs": A["conv_bytes"] / (st_mean[4] / 1e3) / 1e9,
            "peak_gbs": hbm,
            "frac": A["conv_bytes"] / (st_mean[4] / 1e3) / 1e9 / hbm,
            "bytes_per_step": A["conv_bytes"],
        }
        res["roofline"]["traffic"] = None  # the committed capture is of the conv-less value phase
    if args.fp8:
        res["config"]["workload"] += (" + FP8 projections (E4M3 e and W, power-of-two scales per "
                                      "row and output channel, fp32 accumulation)")
        res["roofline"]["kernel"] = res["roofline"]["kernel"].replace("(tcgen05", "(tcgen05 kind::f8f6f4")
        res["roofline"]["traffic"] = kernel_traffic("traffic_fp8.json")
    if args.rows_target:
        res["config"]["workload"] += " [profiling variant: tables of %d rows]" % args.rows_target
    if args.workload != "prefill_bf16":
        # the committed captures: the prefill shapes, and the decode workload's one launch
        res["roofline"]["traffic"] = (
            kernel_traffic("traffic_decode.json", "dram_bytes_per_launch")
            if args.workload == "decode_mb" and short_fused and not args.rows_target else None)
    if not args.no_cpu_baseline and world == 1:
        res["cpu_baseline"] = cpu_baseline(P, args.cpu_seconds)
    return res


# ---------------------------------------------------------- backward leg

def run_backward_bench(args, rank, world, dist):
    """The backward step on the same workload: dh, dW_K, dW_V, dnorm_q,
    dnorm_k and the fp32 table gradients (accumulated) for a seeded dL/dout."""
    import torch
    from hashed_gram_embedding_compress_b200 import synth

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    P = setup(rank, device, args.rows_target, args.workload)
    sh, m, h = P["sh"], P["m"], P["h"]
    R, M, d, dm = sh.rows_out, sh.branches, sh.d_hidden, sh.d_mem
    tok_d = P["tokens"].to(device)
    dout = synth.make_grad_out(sh, P["seeds"], device=device)
    dh = torch.empty_like(h)
    g = dict(dw_k=torch.zeros((M, d, dm), device=device), dw_v=torch.zeros((d, dm), device=device),
             dnorm_q=torch.zeros((M, d), device=device), dnorm_k=torch.zeros((M, d), device=device),
             dtables=[torch.zeros((int(p), sh.d_head), device=device) for p in P["primes"]])
    stream = torch.cuda.current_stream()

    from hashed_gram_embedding_compress_b200 import dp

    def step():
        m.backward(tok_d, h, dout, dh, t_begin=sh.t_begin, stream=stream, **g)
        if dist:
            # data-parallel replicas: the dense gradients are summed over the ranks
            dp.all_reduce_dense([g["dw_k"], g["dw_v"], g["dnorm_q"], g["dnorm_k"]])

    clk = ClockSampler(local).__enter__()
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if m.check_errors(stream) != 0:
        raise RuntimeError("device error during warm-up")
    t_load = time.monotonic()
    while time.monotonic() - t_load < args.load_seconds:
        for _ in range(5):
            step()
        torch.cuda.synchronize()
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(K)]
    for row in evs:
        for ev in row:
            ev.record(stream)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = m.kernel_launches()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t0.record(stream)
    for k in range(K):
        m.profile_next_backward(evs[k])
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    t_end = time.monotonic()
    time.sleep(0.3)
    clk.__exit__(None, None, None)
    if dist:
        dist.barrier()
    launches = m.kernel_launches() - launches0
    ms = max_over_ranks(t0.elapsed_time(t1), dist, device)
    st = [sum(evs[k][i].elapsed_time(evs[k][i + 1]) for k in range(K)) / K for i in range(5)]
    if m.check_errors(stream) != 0:
        raise RuntimeError("device error during the timed steps")

    # e2e: h and dL/dout in from pinned host memory, dh back, every step
    h_h, g_h = h.cpu().pin_memory(), dout.cpu().pin_memory()
    dh_h = torch.empty_like(h_h).pin_memory()
    tok_h = P["tokens"].pin_memory()

    def e2e_step():
        # through the host-buffer entry point (tokens, h, dout in; dh back)
        m.backward_host(tok_h, h_h, g_h, dh_h, t_begin=sh.t_begin, stream=stream, **g)
        if dist:
            dp.all_reduce_dense([g["dw_k"], g["dw_v"], g["dnorm_q"], g["dnorm_k"]])

    e2e_step()
    torch.cuda.synchronize()
    E = e2e_count(args.e2e_steps, e2e_step, dist)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(E):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, device)
    if rank != 0:
        return None

    hbm, tflops_burst, tflops_sus, peak_kind = load_peaks()
    A = algorithmic(sh)
    gemm_flops = 3 * A["gemm_flops"]       # k, v recomputed; weight gradients; de
    gemm_s = (st[1] + st[3] + st[4]) / 1e3
    elt = 2 if sh.dtype == "bf16" else 4
    # gate backward: h, dout, k and v (fp32) read; dh and [dk dv] written
    gate_bytes = R * (2 * M * d * elt + 4 * (M + 1) * d + M * d * elt + (M + 1) * d * elt)
    return {
        "metric": "Engram backward tokens/s (gradients of h, W_K, W_V, RMSNorm weights, tables)",
        "value": R * world * K / (ms / 1e3), "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": max(3, args.warmup), "ms_per_step": ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": sh.dtype, "data": "synthetic",
        "config": {"workload": DESCRIBE[args.workload] + " [backward step, dL/dout ~ N(0, 1)]",
                   "global_batch": R * world, "seq_len": sh.T,
                   "parallelism": "replicas" if world > 1 else "single",
                   "l2": "no flush: inputs larger than L2"},
        "roofline": {"kernel": "the library's tcgen05 contractions of the backward "
                               "(gemm_pair_kernel: k and v recomputed; dW; de)",
                     "bound": "tensor", "achieved": gemm_flops / gemm_s / 1e12,
                     "peak": tflops_burst, "unit": "TFLOP/s",
                     "frac": gemm_flops / gemm_s / 1e12 / tflops_burst, "traffic": None,
                     "peak_source": "%s bf16 burst (cuBLAS, best of 10)" % peak_kind,
                     "peak_sustained": tflops_sus,
                     "frac_of_sustained": gemm_flops / gemm_s / 1e12 / tflops_sus},
        "gate_backward": {"kernel": "gate_backward_kernel + dnorm_reduce_kernel", "bound": "hbm",
                          "achieved_gbs": gate_bytes / (st[2] / 1e3) / 1e9, "peak_gbs": hbm,
                          "frac": gate_bytes / (st[2] / 1e3) / 1e9 / hbm,
                          "bytes_per_step": gate_bytes},
        "stages_ms": {"hash_gather": st[0], "kv_recompute": st[1], "gate_backward": st[2],
                      "weight_grads": st[3], "de_and_table_grads": st[4]},
        "e2e": {"value": R * world * E / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": tok_h.numel() * 4 + 2 * h_h.numel() * h_h.element_size(),
                "d2h_bytes_per_step": dh_h.numel() * dh_h.element_size(), "steps": E,
                "path": "engram_backward_host: C ABI call on pinned host buffers (tokens, h, "
                        "dL/dout in; dh back), copies inside the timed region"},
        "gpu_launches": launches,
        "clocks": dict(clk.summary(t_load + 0.5, t_end + 0.15),
                       window="last 1 s of back-to-back warm-up steps and the timed steps"),
    } | ({"cpu_baseline": cpu_baseline_backward(P, dout, args.cpu_seconds)}
         if not args.no_cpu_baseline and world == 1 else {})


# ------------------------------------------------------ host-offload leg

def run_offload(args):
    """Tables in page-locked host memory (section 2.5, Figure 2b).

    Per step: engram_prefetch of the NEXT step's tokens on a side stream (hash,
    de-duplicate, copy each distinct row once over PCIe into HBM staging),
    while the main stream runs the backbone stand-in (4096^3 bf16 GEMMs) and
    the engram forward of the current step from the staged rows."""
    import torch
    from hashed_gram_embedding_compress_b200 import engram as eg
    from hashed_gram_embedding_compress_b200 import synth

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    sh0 = synth.SHAPES["offload"]
    row_bytes = sh0.d_head * 2
    sh = sh0.replace(rows_target=int(args.offload_gb * 1e9 / (sh0.num_tables * row_bytes)))
    seeds = synth.stream_seeds(sh)
    comp_map = synth.make_comp_map(sh, seeds)
    hash_seed = synth.make_hash_seed(seeds)
    m = eg.Engram(eg.make_config(vocab=sh.vocab, cvocab=sh.cvocab, comp_map=comp_map,
                                 orders=sh.orders, heads=sh.heads, d_head=sh.d_head,
                                 d_hidden=sh.d_hidden, branches=sh.branches, dtype=sh.dtype,
                                 table_rows_target=sh.rows_target, hash_seed=hash_seed,
                                 table_location="pinned_host"))
    primes, _ = m.hash_params()
    # pageable buffers, then page-locked and mapped into the device's address space
    t_setup = time.time()
    cudart = torch.cuda.cudart()
    g = torch.Generator(device=dev)
    g.manual_seed(seeds["tables"])
    tables = []
    try:
        for p in primes.tolist():
            t = torch.empty((p, sh.d_head), dtype=torch.bfloat16)
            rc = cudart.cudaHostRegister(t.data_ptr(), t.numel() * 2, 3)  # portable | mapped
            if int(rc) != 0:
                raise RuntimeError("cudaHostRegister failed (%s)" % rc)
            tables.append(t)
            step = 1 << 22
            for a in range(0, p, step):
                b = min(p, a + step)
                x = torch.randn((b - a, sh.d_head), generator=g, device=dev).mul_(0.02)
                t[a:b].copy_(x.to(torch.bfloat16))
        torch.cuda.synchronize()
        t_setup = time.time() - t_setup
        w_k, w_v, nq, nk = [x.to(dev) for x in synth.make_weights(sh, seeds)]
        m.set_params(tables, w_k, w_v, nq, nk)
        h = synth.make_hidden(sh, seeds, device=dev)
        K = max(3, args.steps)
        toks = [synth.make_tokens(sh, synth.stream_seeds(sh, extra=100 + k)).to(dev)
                for k in range(K + 2)]
        m.reserve(sh.rows_out)
        t_hot = 0.0
        if args.hot_rows > 0:
            # calibration: the rows four other batches of the same token
            # distribution address most often
            calib = torch.cat([synth.make_tokens(sh, synth.stream_seeds(sh, extra=1000 + c))
                               for c in range(4)]).to(dev)
            t0 = time.time()
            m.build_hot_cache(calib, args.hot_rows)
            t_hot = time.time() - t0
        a_ = torch.randn(4096, 4096, device=dev, dtype=torch.bfloat16)
        b_ = torch.randn(4096, 4096, device=dev, dtype=torch.bfloat16)
        main = torch.cuda.current_stream()
        side = torch.cuda.Stream()
        ev = lambda: torch.cuda.Event(enable_timing=True)

        def timed(fn, stream, reps):
            e0, e1 = ev(), ev()
            e0.record(stream)
            for i in range(reps):
                fn(i)
            e1.record(stream)
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) / reps

        pcie = pcie_peak_gbs(dev)
        for _ in range(3):
            a_ @ b_
        t_gemm = timed(lambda i: a_ @ b_, main, 20)

        def measure(route):
            """One route of the prefetch's copy: alone, then pipelined."""
            m.set_prefetch(*route)
            # the prefetch alone (host clock from the call until its rows are
            # staged), then the forward from the staged rows (CUDA events)
            uniq, t_pf, t_fw, hits = [], [], [], []
            for k in range(K):
                torch.cuda.synchronize()
                w0 = time.perf_counter()
                m.prefetch(toks[k], stream=side)
                m.prefetch_wait()
                t_pf.append((time.perf_counter() - w0) * 1e3)
                f0, f1 = ev(), ev()
                f0.record(main)
                m.forward(toks[k], h, h, stream=main)
                f1.record(main)
                torch.cuda.synchronize()
                t_fw.append(f0.elapsed_time(f1))
            for k in range(3):
                uniq.append(m.prefetch(toks[k], stream=side, want_count=True))
                hits.append(m.prefetch_hot_hits())
                m.forward(toks[k], h, h, stream=main)
                torch.cuda.synchronize()
            t_pf, t_fw = statistics.median(t_pf[1:]), statistics.median(t_fw[1:])
            n_hide = max(1, int(-(-(t_pf - t_fw) // t_gemm)))  # GEMMs whose time covers it

            def pipeline(n_gemm):
                m.prefetch(toks[0], stream=side)
                torch.cuda.synchronize()
                e0, e1 = ev(), ev()
                e0.record(main)
                for k in range(K):
                    m.prefetch(toks[k + 1], stream=side)  # next step's rows, overlapped
                    for _ in range(n_gemm):
                        a_ @ b_
                    m.forward(toks[k], h, h, stream=main)
                e1.record(main)
                torch.cuda.synchronize()
                m.forward(toks[K], h, h, stream=main)  # consume the last pending prefetch
                torch.cuda.synchronize()
                return e0.elapsed_time(e1) / K

            t_pipe1 = pipeline(1)
            t_pipe_n = pipeline(n_hide)
            if m.check_errors() != 0:
                raise RuntimeError("device error in the offload run")
            u, hot = statistics.mean(uniq), statistics.mean(hits)
            pcie_bytes = (u - hot) * row_bytes
            compute_n = n_hide * t_gemm + t_fw
            serial_n = t_pf + compute_n
            return {
                "route": route[0], "workers": route[1] or "default",
                "unique_rows_per_step": u,
                "unique_fraction": u / (sh.rows_out * sh.num_tables),
                "pcie_bytes_per_step": pcie_bytes,
                "prefetch_ms": t_pf,
                "pcie_gbs": pcie_bytes / (t_pf / 1e3) / 1e9,
                "pcie_frac_of_peak": pcie_bytes / (t_pf / 1e3) / 1e9 / pcie,
                "forward_from_staging_ms": t_fw,
                "step_ms_1_gemm": t_pipe1,
                "serial_ms_1_gemm": t_pf + t_gemm + t_fw,
                "gemms_to_hide_prefetch": n_hide,
                "step_ms_n_gemm": t_pipe_n,
                "serial_ms_n_gemm": serial_n,
                "loss_vs_hidden_prefetch": t_pipe_n / compute_n - 1.0,
                # 1: the shorter of prefetch and compute fully hidden; 0: serial
                "overlap_fraction": (serial_n - t_pipe_n) / min(t_pf, compute_n),
                "hot_hits_per_step": hot,
            }

        routes = [measure(("host_threads", 0)), measure(("zero_copy", 0)),
                  measure(("zero_copy", 16))]
        best = min(routes, key=lambda r: r["step_ms_1_gemm"])
        total_bytes = sum(t.numel() * 2 for t in tables)
        return {
            "metric": METRIC, "value": sh.rows_out / (best["step_ms_1_gemm"] / 1e3),
            "unit": "tokens/s", "n_gpus": 1, "steps": K, "warmup": 1,
            "ms_per_step": best["step_ms_1_gemm"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": DESCRIBE["offload"], "global_batch": sh.rows_out,
                       "seq_len": sh.T, "parallelism": "single",
                       "host_tables_gb": total_bytes / 1e9,
                       "rows_per_table": primes.tolist(),
                       "host_cores": len(os.sched_getaffinity(0))},
            "offload": {
                "route": best["route"],
                "pcie_peak_gbs": pcie,
                "pcie_peak_how": "pinned 1 GiB host-to-device copy, best of 10 (CUDA events)",
                "standin_gemm_ms": t_gemm,
                "routes": routes,
                "host_setup_s": t_setup,
                "hot_cache": {
                    "rows": args.hot_rows,
                    "gb": args.hot_rows * row_bytes / 1e9,
                    "build_s": t_hot,
                    "hit_fraction": best["hot_hits_per_step"] / best["unique_rows_per_step"]
                    if best["unique_rows_per_step"] else 0.0,
                },
            },
        }
    finally:
        torch.cuda.synchronize()
        for t in tables:
            cudart.cudaHostUnregister(t.data_ptr())


def pcie_peak_gbs(dev) -> float:
    """Host-to-device copy rate of this machine: a pinned 1 GiB buffer, best of 10."""
    import torch
    src = torch.empty(1 << 30, dtype=torch.uint8).pin_memory()
    dst = torch.empty(1 << 30, dtype=torch.uint8, device=dev)
    best = None
    for _ in range(10):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        dst.copy_(src, non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        t = e0.elapsed_time(e1)
        best = t if best is None else min(best, t)
    del src, dst
    return (1 << 30) / (best / 1e3) / 1e9


# ----------------------------------------------------------- CPU oracle leg

def cpu_baseline(P, budget_s: float):
    """The oracle, as it stands, on a bounded sample of the same workload.

    Compress + hash run on every position; gather, projections and gate on
    the first n rows, n grown until the sample takes about `budget_s` seconds.
    tokens/s = 1 / (hash time per position + gather+fp time per row)."""
    import numpy as np
    import torch

    import oracle

    sh = P["sh"]
    tokens = P["tokens"].numpy()
    t0 = time.perf_counter()
    c, z, mult, primes = oracle.forward_indices(tokens, P["comp_map"].numpy(), sh.cvocab,
                                                sh.orders, sh.heads, P["hash_seed"],
                                                sh.rows_target, t_begin=sh.t_begin)
    t_hash = (time.perf_counter() - t0) / sh.rows_out

    def to_np(t):
        t = t.detach().contiguous().cpu()
        return t.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.numpy()

    wk, wv = to_np(P["w_k"]), to_np(P["w_v"])
    nq, nk = P["nq"].cpu().numpy(), P["nk"].cpu().numpy()
    # FP8 projections: W quantised once, as the library does when they are switched on
    w8 = oracle.quantize_weights_e4m3(wk, wv) if P.get("fp8") else None
    n, spent, total_rows, total_t = 8, 0.0, 0, 0.0
    while spent < budget_s and total_rows < sh.rows_out:
        rows = np.arange(total_rows, min(sh.rows_out, total_rows + n))
        zr = z[rows]
        mini = [to_np(t[torch.from_numpy(zr[:, s]).to(t.device)]) for s, t in enumerate(P["tables"])]
        zz = np.tile(np.arange(len(rows))[:, None], (1, sh.num_tables))
        hr = to_np(P["h"][torch.from_numpy(rows).to(P["h"].device)])
        t0 = time.perf_counter()
        e = oracle.gather(mini, zz)
        want = P["conv"] is not None
        if w8 is not None:
            _, delta, _ = oracle.project_gate_fp8(e, wk, wv, nq, nk, hr, 1e-6, want_delta=want,
                                                  weights=w8)
        else:
            _, delta, _ = oracle.project_gate(e, wk, wv, nq, nk, hr, 1e-6, want_delta=want)
        if P["conv"] is not None:
            # Eq. 5 over the sample's positions (consecutive rows of one sequence)
            cw, nw, W, dil = P["conv"]
            for mb in range(sh.branches):
                y = oracle.short_conv(delta[:, mb], cw.cpu().numpy(), nw.cpu().numpy(), dil, 1e-6)
                oracle.add_round(np.ascontiguousarray(hr[:, mb]), y)
        dt = time.perf_counter() - t0
        total_rows += len(rows)
        total_t += dt
        spent += dt
        n *= 2
    per_row = t_hash + total_t / total_rows
    return {"value": 1.0 / per_row, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": "compress+hash on all %d positions; gather+%sprojection+gate%s on the first "
                      "%d rows (%.1f s); single-threaded C, fp64" % (
                          sh.rows_out, "E4M3 quantisation+" if w8 is not None else "",
                          "+short conv" if P["conv"] is not None else "", total_rows, total_t)}


def cpu_baseline_backward(P, dout, budget_s: float):
    """The oracle's backward, as it stands, on a bounded sample of the same
    workload: compress + hash on every position; gather, the exact derivative
    and the table-gradient scatter on the first n rows, n grown until the
    sample takes about `budget_s` seconds.  tokens/s as in cpu_baseline."""
    import numpy as np
    import torch

    import oracle

    sh = P["sh"]
    t0 = time.perf_counter()
    c, z, mult, primes = oracle.forward_indices(P["tokens"].numpy(), P["comp_map"].numpy(),
                                                sh.cvocab, sh.orders, sh.heads, P["hash_seed"],
                                                sh.rows_target, t_begin=sh.t_begin)
    t_hash = (time.perf_counter() - t0) / sh.rows_out

    def to_np(t):
        t = t.detach().contiguous().cpu()
        return t.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.numpy()

    wk, wv = to_np(P["w_k"]), to_np(P["w_v"])
    nq, nk = P["nq"].cpu().numpy(), P["nk"].cpu().numpy()
    n, total_rows, total_t = 4, 0, 0.0
    while total_t < budget_s and total_rows < sh.rows_out:
        rows = np.arange(total_rows, min(sh.rows_out, total_rows + n))
        zr = z[rows]
        mini = [to_np(t[torch.from_numpy(zr[:, s]).to(t.device)]) for s, t in enumerate(P["tables"])]
        zz = np.tile(np.arange(len(rows))[:, None], (1, sh.num_tables))
        rs = torch.from_numpy(rows)
        hr = to_np(P["h"][rs.to(P["h"].device)])
        gr = dout[rs.to(dout.device)].double().cpu().numpy()
        t0 = time.perf_counter()
        e = oracle.gather(mini, zz)
        b = oracle.backward(e, wk, wv, nq, nk, hr, gr, 1e-6, round_dkv=sh.dtype == "bf16")
        oracle.table_grad(b["de"], zz, [len(rows)] * sh.num_tables, sh.d_head)
        total_t += time.perf_counter() - t0
        total_rows += len(rows)
        n *= 2
    per_row = t_hash + total_t / total_rows
    return {"value": 1.0 / per_row, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": "compress+hash on all %d positions; gather+backward+table scatter on the "
                      "first %d rows (%.1f s); single-threaded C, fp64" % (
                          sh.rows_out, total_rows, total_t)}


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle, as it stands, on this arm's workload.

    Inputs are drawn exactly as for the library's arm (tables on the GPU with
    the same seeded generator, table sizes from the oracle's own prime
    sequence) without loading the library.  Each step is a bounded sample of
    the workload (compress + hash of every position, the floating-point steps
    on a prefix of rows), timed on one host core."""
    if rank != 0:
        return None
    import torch

    import oracle
    from hashed_gram_embedding_compress_b200 import synth

    local = int(os.environ.get("LOCAL_RANK", "0"))
    device = torch.device("cpu")
    if torch.cuda.is_available():
        torch.cuda.set_device(local)
        device = torch.device("cuda", local)
    sh0 = synth.SHAPES[args.workload]
    target = args.rows_target or sh0.rows_target
    primes = oracle.table_primes(target, sh0.num_tables)
    P = draw_inputs(0, device, primes, args.rows_target, args.workload,
                    args.short_conv) | dict(fp8=args.fp8)
    sh = P["sh"]
    budget = max(1.0, min(args.cpu_seconds, 120.0 / max(1, args.steps + args.warmup)))
    if args.backward:
        dout = synth.make_grad_out(sh, P["seeds"], device=P["h"].device)
        leg = lambda: cpu_baseline_backward(P, dout, budget)  # noqa: E731
        metric = "Engram backward tokens/s (gradients of h, W_K, W_V, RMSNorm weights, tables)"
    else:
        leg = lambda: cpu_baseline(P, budget)  # noqa: E731
        metric = METRIC
    for _ in range(args.warmup):
        leg()
    vals, walls = [], []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        vals.append(leg())
        walls.append(time.perf_counter() - t0)
    v = statistics.median(x["value"] for x in vals)
    return {
        "impl": "reference", "metric": metric, "value": v, "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup,
        # one step is the bounded sample below, not the whole batch
        "ms_per_step": statistics.median(walls) * 1e3,
        "ms_per_full_batch_at_this_rate": sh.rows_out / v * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": DESCRIBE.get(args.workload, args.workload),
                   "global_batch": sh.rows_out, "seq_len": sh.T, "parallelism": "single",
                   "step": "a bounded sample of the batch: " + vals[-1]["sample"]},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": vals[-1]["sample"]},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    dist = None
    if world > 1 and args.impl == "ours":
        import datetime

        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    if args.impl == "reference":
        res = run_reference(args, rank, world)
    elif args.workload == "offload":
        res = run_offload(args) if rank == 0 else None
    elif args.backward:
        res = run_backward_bench(args, rank, world, dist)
    else:
        res = run_ours(args, rank, world, dist)
    if res is not None:
        print(json.dumps(res), flush=True)
    if dist:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
