#!/usr/bin/env python
"""Benchmark of the hybrid CSA/HCA attention step on B200.

Headline (one JSON line on rank 0): CSA decode at 128K context -- batch 8, one
query per sequence at position 131071, m = 4 (32768 compressed entries), 64x128
indexer, top-k 1024, 128 heads x 512, window 128.  A step is one pass of the
decode hot path over the resident cache: csa_decode_step, i.e. csa_index ->
csa_topk -> csa_attend (+ split combine) with the top-k and attention kernels
launched as programmatic dependents; the K timed steps are one CUDA graph.  Six decode
states rotate (each has 79 MB of step inputs; 5 x 79 MB pass through the
126 MB L2 between two uses of one state), so no step finds its inputs in L2
and no flush is needed between steps.

The same run also measures the other synthetic workloads (prefill chunk,
HCA decode at 1M, FP4-indexer decode at 1M, cache compression) and reports them
under "workloads".

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--no-extra]

With N > 1 (torchrun, one rank per GPU) every rank runs its own independent
batch (weak scaling); the only collectives are a barrier and a max-reduction of
the timings.  `--impl reference` times the float64 CPU oracle on a bounded
sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from long_context_compressed_06_b200 import workloads as W  # noqa: E402

L2_FLUSH_BYTES = 256 << 20
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
PROFILES = os.path.join(ROOT, "profiles")
METRIC = "CSA decode queries/s @128K ctx + HBM GB/s vs peak; prefill TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- distributed plumbing
def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), \
        int(os.environ.get("LOCAL_RANK", "0"))


def dist_init(world: int, backend: str = "nccl"):
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=180))


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    """Max of a per-rank scalar (the job time is the slowest rank's)."""
    if world == 1:
        return float(x)
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank_step: int, steps: int, world: int, t_max: float) -> float:
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    return units_per_rank_step * steps * world / t_max


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own independent batch."""
    return base_seed + 7919 * rank


# ----------------------------------------------------------------------------- peaks, clocks, profiles
def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while timing runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path:
            return None
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[4:]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r[1:5]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


def kernel_source_hash(*names) -> str:
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "long_context_compressed_06_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(summary_name: str, src_hash: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on this kernel source."""
    path = os.path.join(PROFILES, summary_name)
    try:
        text = open(path).read()
    except OSError:
        return None
    mh = re.search(r"kernel_source_hash:\s*([0-9a-f]+)", text)
    mt = re.search(r"dram_bytes_per_launch:\s*([0-9,]+)", text)
    if not mh or not mt or mh.group(1) != src_hash:
        return None
    return int(mt.group(1).replace(",", ""))


# ----------------------------------------------------------------------------- timing helpers
class Timer:
    """Per-step CUDA-event timing on the current stream with an L2 flush and a
    short device sleep before each step (both outside the timed interval; the
    sleep lets the host enqueue the step before the GPU reaches it)."""

    def __init__(self, device):
        self.flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)

    def prep(self):
        self.flush.fill_(1)
        torch.cuda._sleep(2_000_000)

    def run(self, fn, steps: int, warmup: int, marks: int = 0):
        """Runs fn() warmup+steps times; fn calls mark(0..marks-1) between its kernels.
        Returns (total seconds of the timed steps, the marks+1 segment times averaged)."""
        for _ in range(warmup):
            self.prep()
            fn(lambda i: None)
        torch.cuda.synchronize()
        tot = 0.0
        seg = [0.0] * (marks + 1)
        for _ in range(steps):
            self.prep()
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(marks + 2)]
            evs[0].record()
            fn(lambda i: evs[1 + i].record())
            evs[-1].record()
            torch.cuda.synchronize()
            tot += evs[0].elapsed_time(evs[-1]) / 1e3
            if marks:
                for i in range(marks + 1):
                    seg[i] += evs[i].elapsed_time(evs[i + 1]) / 1e3
        return tot, [s / max(steps, 1) for s in seg]


# ----------------------------------------------------------------------------- CSA decode (headline)
def csa_decode_state(csa, wl: W.Workload, device, seed: int):
    wl = wl.scaled(seed=seed)
    L = W.pool_logits(wl, device)
    A = torch.empty((wl.batch, wl.T, wl.D), dtype=torch.bfloat16, device=device)
    B = torch.empty_like(A)
    for b in range(wl.batch):
        A[b] = W.stream(wl, "A", b, device)
        B[b] = W.stream(wl, "B", b, device)
    C = csa.csa_compress(A, B, L, wl.m, True, None, wl.eps)
    del B
    st = dict(wl=wl, A=A, C=C, L=L,
              qI=W.index_queries(wl, device), w=W.index_weights(wl, device), kI=W.index_keys(wl, device),
              q=W.queries(wl, device), qp=wl.q_positions().to(device))
    st["S"] = torch.empty((wl.batch, wl.nq, wl.N), dtype=torch.float32, device=device)
    st["idx"] = torch.empty((wl.batch, wl.nq, wl.k), dtype=torch.int32, device=device)
    st["out"] = torch.empty_like(st["q"])
    nws = csa.attend_workspace_bytes(wl.batch, wl.nq, wl.H, wl.D, wl.k + wl.W)
    st["ws"] = torch.empty(max(nws, 16), dtype=torch.uint8, device=device)
    st["launches"] = 3 + (1 if nws > 0 else 0)
    return st


def decode_cache_state(csa, wl: W.Workload, device, seed: int):
    """A decode state that keeps only the last W rows of stream A (the window
    cache a decode loop holds) instead of the whole stream."""
    st = csa_decode_state(csa, wl, device, seed)
    st["win"] = st["A"][:, wl.T - wl.W:].contiguous()
    st["win_pos0"] = wl.T - wl.W
    del st["A"]
    return st


def decode_step(csa, st):
    """One decode step through the public API: csa_decode_step (csa_index ->
    csa_topk -> csa_attend, the last two launched as programmatic dependents)."""
    wl = st["wl"]
    csa.csa_decode_step(st["qI"], st["w"], st["kI"], st["q"], st["C"], st.get("win", st.get("A")), st["qp"], wl.m,
                        wl.k, wl.W, wl.scale, wl.eps, scores=st["S"], idx=st["idx"], out=st["out"],
                        workspace=st["ws"], win_pos0=st.get("win_pos0", 0))


def index_bytes(wl: W.Workload, fp4=False) -> int:
    """Algorithmic bytes of one indexer launch: keys, queries, weights in; scores out."""
    if fp4:
        kb = wl.N * (wl.d_I // 2 + wl.d_I // 16)
        qb = wl.nq * wl.H_I * (wl.d_I // 2 + wl.d_I // 16)
    else:
        kb = wl.N * wl.d_I * 2
        qb = wl.nq * wl.H_I * wl.d_I * 2
    return wl.batch * (kb + qb + wl.nq * wl.H_I * 4 + wl.nq * wl.N * 4)


def decode_step_bytes(wl: W.Workload) -> int:
    """Algorithmic HBM bytes of one decode step (per query: indexer keys, q_I, w,
    gathered entries, window rows, q, output, indices)."""
    per_q = (wl.N * wl.d_I * 2 + wl.H_I * wl.d_I * 2 + wl.H_I * 4 + wl.k * wl.D * 2 + wl.W * wl.D * 2
             + 2 * wl.H * wl.D * 2 + wl.k * 4)
    return wl.batch * wl.nq * per_q


DEVICE_STATES = 6


def bench_csa_decode(csa, args, device, world, rank, peaks):
    """The headline: the 128K decode step.  The K timed steps are captured in
    one CUDA graph (as consecutive attention layers of a decode forward would
    be), each step complete before the next starts, and replayed once between
    two events on the launch stream.  DEVICE_STATES states (each 79 MB of step
    inputs, together more than the 126 MB L2) rotate, so every step reads its
    keys and rows from HBM without an L2 flush between steps (a write flush
    would leave dirty lines whose write-back shares DRAM with the step)."""
    wl = W.CSA_DECODE
    states = [decode_cache_state(csa, wl, device, rank_seed(0 if i == 0 else 101 + i, rank))
              for i in range(DEVICE_STATES)]
    st = states[0]
    for S in states:
        decode_step(csa, S)  # eager first (lazy initialisation outside the capture)
    torch.cuda.synchronize()

    def capture(n, first):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(first, first + n):
                decode_step(csa, states[i % len(states)])
        return g

    g_warm, g_timed = capture(args.warmup, 0), capture(args.steps, args.warmup)
    graphs = [g_warm, g_timed]
    torch.cuda.synchronize()
    g_warm.replay()
    torch.cuda.synchronize()
    barrier(world)
    with ClockSampler(torch.cuda.current_device()) as clk:
        t0 = time.perf_counter()
        torch.cuda._sleep(2_000_000)  # lets the host enqueue ahead of the GPU (outside the events)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g_timed.replay()
        e1.record()
        torch.cuda.synchronize()
        t_graph = e0.elapsed_time(e1) / 1e3
        # keep the GPU under the same load until the sampler has seen >= 1 s of it
        while time.perf_counter() - t0 < 1.5:
            for _ in range(5):
                g_timed.replay()
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    t_max = max_over_ranks(t_graph, world, device)
    value = job_rate(wl.batch * wl.nq, args.steps, world, t_max)
    # per-kernel breakdown: each kernel of the step launched n times over the
    # rotation inside one graph, between two events on the launch stream
    seg = kernel_breakdown(csa, states, args)
    t_index = seg[0]
    idx_bytes = index_bytes(wl)
    src_hash = kernel_source_hash("index_tc.cu", "tc.cuh")
    ach = idx_bytes / t_index / 1e9
    roof = {"kernel": "csa_index", "bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4),
            "traffic": profiled_traffic("csa_index_decode_128k.md", src_hash),
            "algorithmic_bytes_per_launch": idx_bytes, "launch_ms": round(t_index * 1e3, 4)}
    step_bytes = decode_step_bytes(wl)
    step_s = t_max / args.steps
    del graphs, g_warm, g_timed
    e2e = e2e_csa_decode(csa, states, args, device, world, rank)
    return dict(value=value, ms_per_step=step_s * 1e3, roofline=roof, clocks=clk.summary(), e2e=e2e,
                launches=st["launches"] * args.steps,
                step={"algorithmic_bytes": step_bytes, "hbm_gbs": round(step_bytes / step_s / 1e9, 1),
                      "hbm_frac_of_8tbs": round(step_bytes / step_s / 8e12, 4),
                      "hbm_frac_of_measured": round(step_bytes / step_s / 1e9 / peaks["hbm_gbs"], 4),
                      "kernel_ms": {"csa_index": round(seg[0] * 1e3, 4), "csa_topk": round(seg[1] * 1e3, 4),
                                    "csa_attend+combine": round(seg[2] * 1e3, 4)}}), st


def kernel_breakdown(csa, states, args):
    """Seconds per launch of csa_index, csa_topk and csa_attend (+ its split
    combine) in the decode step: n launches of one kernel, cycling over the
    decode states (inputs larger than L2), captured in one graph and timed by
    events around its replay, so that no graph-launch gap sits between them."""
    n = max(args.steps, 6)
    n = (n + len(states) - 1) // len(states) * len(states)

    def launch(k, S):
        wl = S["wl"]
        if k == 0:
            csa.csa_index(S["qI"], S["w"], S["kI"], S["qp"], wl.m, scores=S["S"])
        elif k == 1:
            csa.csa_topk(S["S"], S["qp"], wl.m, wl.k, idx=S["idx"])
        else:
            csa.csa_attend(S["q"], S["C"], S["idx"], S.get("win", S.get("A")), S["qp"], wl.W, wl.scale,
                           wl.eps, out=S["out"], workspace=S["ws"], win_pos0=S.get("win_pos0", 0))

    seg = []
    for k in range(3):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(n):
                launch(k, states[i % len(states)])
        torch.cuda.synchronize()
        for i in range(max(1, args.warmup // 2)):
            g.replay()
        torch.cuda.synchronize()
        torch.cuda._sleep(2_000_000)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        seg.append(e0.elapsed_time(e1) / 1e3 / n)
        del g
    return seg


E2E_STATES = 4


def e2e_csa_decode(csa, states, args, device, world, rank):
    """Same metric through the public API with the step's inputs on the host.
    Every step copies q, q_I, w and q_pos from pinned host memory and reads the
    attention output back.  As a serving loop would, each decode state's step
    (the H2D copies, the csa_decode_step call, the D2H copy) is captured once
    in a CUDA graph; consecutive steps use different
    states, replayed on their own streams, so one step's copies overlap its
    neighbours' kernels.  The states' step inputs (4 x 79 MB) exceed the L2,
    so no step finds its inputs in L2 and no flush is needed between steps."""
    wl = states[0]["wl"]
    names = ("q", "qI", "w", "qp")
    states = states[:E2E_STATES]
    host_in = [{k: s_[k].cpu().pin_memory() for k in names} for s_ in states]
    host_out = [torch.empty(s_["out"].shape, dtype=s_["out"].dtype).pin_memory() for s_ in states]
    h2d = sum(t.numel() * t.element_size() for t in host_in[0].values())
    d2h = host_out[0].numel() * host_out[0].element_size()
    streams = [torch.cuda.Stream(device) for _ in states]

    def body(j):
        S = states[j]
        for k in names:
            S[k].copy_(host_in[j][k], non_blocking=True)
        decode_step(csa, S)
        host_out[j].copy_(S["out"], non_blocking=True)

    graphs = []
    for j in range(len(states)):
        with torch.cuda.stream(streams[j]):
            body(j)  # eager run first (lazy initialisation outside the capture)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=streams[j]):
            body(j)
        graphs.append(g)
    torch.cuda.synchronize()
    main = torch.cuda.current_stream(device)

    def run(n, first):
        for i in range(first, first + n):
            j = i % len(states)
            with torch.cuda.stream(streams[j]):
                graphs[j].replay()

    run(args.warmup, 0)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda._sleep(2_000_000)  # lets the host enqueue every step ahead of the GPU (outside the events)
    e0.record(main)
    for s_ in streams:
        s_.wait_stream(main)
    run(args.steps, args.warmup)
    for s_ in streams:
        main.wait_stream(s_)
    e1.record(main)
    torch.cuda.synchronize()
    t_max = max_over_ranks(e0.elapsed_time(e1) / 1e3, world, device)
    del graphs
    return {"value": job_rate(wl.batch * wl.nq, args.steps, world, t_max), "unit": "queries/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "method": "every step: H2D of its inputs from pinned memory, csa_decode_step (csa_index -> csa_topk -> csa_attend), "
                      "D2H of the output, captured once per decode state in a CUDA graph; %d states rotate on "
                      "%d streams (inputs exceed L2, no flush), so copies overlap neighbouring steps"
                      % (E2E_STATES, E2E_STATES)}


# ----------------------------------------------------------------------------- other workloads
def attend_flops(wl: W.Workload, n_keys_per_query) -> float:
    return float(sum(n_keys_per_query)) * wl.H * wl.D * 2 * 2


def bench_prefill(csa, args, device, peaks):
    wl = W.CSA_PREFILL
    A, B = W.streams(wl, device)
    L = W.pool_logits(wl, device)
    C = csa.csa_compress(A, B, L, wl.m)
    del B
    qI, w, kI = W.index_queries(wl, device), W.index_weights(wl, device), W.index_keys(wl, device)
    q = W.queries(wl, device)
    qp = wl.q_positions().to(device)
    S = torch.empty((1, wl.nq, wl.N), dtype=torch.float32, device=device)
    idx = torch.empty((1, wl.nq, wl.k), dtype=torch.int32, device=device)
    out = torch.empty_like(q)
    nws = csa.attend_workspace_bytes(1, wl.nq, wl.H, wl.D, wl.k + wl.W)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=device)

    def step(mark):
        csa.csa_index(qI, w, kI, qp, wl.m, scores=S)
        mark(0)
        csa.csa_topk(S, qp, wl.m, wl.k, idx=idx)
        mark(1)
        csa.csa_attend(q, C, idx, A, qp, wl.W, wl.scale, wl.eps, out=out, workspace=ws)

    steps = max(2, min(args.steps, 5))
    tot, seg = Timer(device).run(step, steps, 2, marks=2)
    pos = list(range(wl.q_pos0, wl.q_pos0 + wl.nq))
    nvis = [min(wl.N, (t + 1) // wl.m) for t in pos]
    idx_flops = float(sum(nvis)) * wl.H_I * wl.d_I * 2
    keys = [min(wl.k, nv) + min(wl.W, t + 1) for t, nv in zip(pos, nvis)]
    att_flops = attend_flops(wl, keys)
    peak = peaks["bf16_tflops"]
    return {"workload": wl.name, "tokens_per_s": wl.nq * steps / tot, "ms_per_step": tot / steps * 1e3,
            "index": {"tflops": round(idx_flops / seg[0] / 1e12, 2), "frac": round(idx_flops / seg[0] / 1e12 / peak, 4),
                      "ms": round(seg[0] * 1e3, 3), "flop": idx_flops},
            "topk_ms": round(seg[1] * 1e3, 3),
            "attend": {"tflops": round(att_flops / seg[2] / 1e12, 2),
                       "frac": round(att_flops / seg[2] / 1e12 / peak, 4), "ms": round(seg[2] * 1e3, 3),
                       "flop": att_flops},
            "peak_tflops": peak, "peak_kind": "bf16 dense, burst"}


def bench_compress(csa, args, device, peaks, wl: W.Workload, seqs: int = 2):
    """Cache build throughput (tokens/s) on `seqs` sequences of the workload's length."""
    L = W.pool_logits(wl, device)
    A = torch.empty((1, wl.T, wl.D), dtype=torch.bfloat16, device=device)
    B = torch.empty_like(A)
    A[0] = W.stream(wl, "A", 0, device)
    B[0] = W.stream(wl, "B", 0, device)
    out = torch.empty((1, wl.N, wl.D), dtype=torch.bfloat16, device=device)
    steps = max(2, min(args.steps, 5))
    tot, _ = Timer(device).run(lambda mark: csa.csa_compress(A, B, L, wl.m, out=out), steps, 2)
    byts = 2 * wl.T * wl.D * 2 + wl.N * wl.D * 2
    t = tot / steps
    return {"workload": wl.name + "_compress", "tokens_per_s": wl.T / t, "ms": round(t * 1e3, 3),
            "hbm_gbs": round(byts / t / 1e9, 1), "frac": round(byts / t / 1e9 / peaks["hbm_gbs"], 4)}


def bench_compress_dynamic(csa, args, device, peaks, wl: W.Workload):
    """Cache build with input-dependent compression weights (tokens/s), one sequence of the workload's
    length: streams A, B and weight rows Z_a, Z_b read once, entries written once."""
    L = W.pool_logits(wl, device)
    A, B, Za, Zb = (torch.empty((1, wl.T, wl.D), dtype=torch.bfloat16, device=device) for _ in range(4))
    A[0] = W.stream(wl, "A", 0, device)
    B[0] = W.stream(wl, "B", 0, device)
    Za[0] = W.compression_weights(wl, "Za", 0, device)
    Zb[0] = W.compression_weights(wl, "Zb", 0, device)
    out = torch.empty((1, wl.N, wl.D), dtype=torch.bfloat16, device=device)
    steps = max(2, min(args.steps, 5))
    tot, _ = Timer(device).run(lambda mark: csa.csa_compress_dynamic(A, B, Za, Zb, L, wl.m, out=out), steps, 2)
    byts = 4 * wl.T * wl.D * 2 + wl.N * wl.D * 2
    t = tot / steps
    return {"workload": wl.name + "_compress_dynamic", "tokens_per_s": wl.T / t, "ms": round(t * 1e3, 3),
            "hbm_gbs": round(byts / t / 1e9, 1), "frac": round(byts / t / 1e9 / peaks["hbm_gbs"], 4)}


def bench_fp8kv_decode(csa, args, device, peaks):
    """The 128K decode attention with the KV cache in FP8 (compressed entries and window rows as e4m3 codes
    plus one exponent byte per 128 channels), timed beside the bf16 attention on the same selection."""
    wl = W.CSA_DECODE
    st = decode_cache_state(csa, wl, device, 0)
    kv8, kv8e = csa.csa_quantize_fp8_kv(st["C"])
    w8, w8e = csa.csa_quantize_fp8_kv(st["win"])
    csa.csa_index(st["qI"], st["w"], st["kI"], st["qp"], wl.m, scores=st["S"])
    csa.csa_topk(st["S"], st["qp"], wl.m, wl.k, idx=st["idx"])
    args8 = (st["q"], kv8, kv8e, st["idx"], w8, w8e, st["qp"], wl.W, wl.scale, wl.eps)
    args16 = (st["q"], st["C"], st["idx"], st["win"], st["qp"], wl.W, wl.scale, wl.eps)
    kw = dict(out=st["out"], workspace=st["ws"], win_pos0=st["win_pos0"])
    steps = max(3, min(args.steps, 20))
    t8, _ = Timer(device).run(lambda mark: csa.csa_attend_fp8kv(*args8, **kw), steps, 3)
    t16, _ = Timer(device).run(lambda mark: csa.csa_attend(*args16, **kw), steps, 3)
    t8, t16 = t8 / steps, t16 / steps
    rows = wl.k + wl.W
    byts8 = wl.batch * (rows * (wl.D + wl.D // 128) + 2 * wl.H * wl.D * 2 + wl.k * 4)
    byts16 = wl.batch * (rows * wl.D * 2 + 2 * wl.H * wl.D * 2 + wl.k * 4)
    return {"workload": "csa_decode_128k_fp8kv_attend", "attend_ms_fp8": round(t8 * 1e3, 4),
            "attend_ms_bf16": round(t16 * 1e3, 4), "bytes_fp8": byts8, "bytes_bf16": byts16,
            "hbm_gbs_fp8": round(byts8 / t8 / 1e9, 1), "frac_fp8": round(byts8 / t8 / 1e9 / peaks["hbm_gbs"], 4)}


def bench_hca(csa, args, device, peaks):
    wl = W.HCA_DECODE
    L = W.pool_logits(wl, device)
    C = torch.empty((wl.batch, wl.N, wl.D), dtype=torch.bfloat16, device=device)
    win = torch.empty((wl.batch, wl.W, wl.D), dtype=torch.bfloat16, device=device)
    for b in range(wl.batch):   # stream -> compressed cache -> discard (window rows kept)
        A = W.stream(wl, "A", b, device).unsqueeze(0)
        B = W.stream(wl, "B", b, device).unsqueeze(0)
        csa.csa_compress(A, B, L, wl.m, out=C[b:b + 1])
        win[b] = A[0, wl.T - wl.W:]
        del A, B
    q = W.queries(wl, device)
    qp = wl.q_positions().to(device)
    out = torch.empty_like(q)
    nws = csa.attend_workspace_bytes(wl.batch, 1, wl.H, wl.D, wl.N + wl.W)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=device)
    step = lambda mark: csa.hca_attend(q, C, wl.m, win, qp, wl.W, wl.scale, wl.eps, out=out, workspace=ws,
                                       win_pos0=wl.T - wl.W)
    step(None)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step(None)
    steps = max(2, min(args.steps, 10))
    tot, _ = Timer(device).run(lambda mark: g.replay(), steps, 2)
    t = tot / steps
    nkeys = wl.N + wl.W
    byts = wl.batch * (nkeys * wl.D * 2 + 2 * wl.H * wl.D * 2)
    flops = wl.batch * nkeys * wl.H * wl.D * 4.0
    t_roof = max(byts / (peaks["hbm_gbs"] * 1e9), flops / (peaks["bf16_tflops"] * 1e12))
    return {"workload": wl.name, "queries_per_s": wl.batch / t, "ms_per_step": round(t * 1e3, 4),
            "hbm_gbs": round(byts / t / 1e9, 1), "tflops": round(flops / t / 1e12, 2),
            "frac_of_roofline": round(t_roof / t, 4)}


def bench_fp4(csa, args, device, peaks):
    wl = W.FP4_DECODE
    kI = W.index_keys(wl, device)
    k4, k4s = csa.csa_quantize_fp4(kI)
    # compressed KV rows drawn N(0,1), then RMSNorm'd like every compressed entry:
    # csa_compress with m = 1 and logits (-inf for the B row, 0 for the A row)
    # pools each row with weight 1 alone and applies the RMSNorm
    raw = W.direct_kv(wl, device)
    one = torch.cat([torch.full((1, wl.D), float("-inf"), device=device), torch.zeros((1, wl.D), device=device)])
    C = csa.csa_compress(raw, raw, one, 1)
    del raw
    win = W.normal_bf16((wl.batch, wl.W, wl.D), 424242, device)
    qI, w = W.index_queries(wl, device), W.index_weights(wl, device)
    q = W.queries(wl, device)
    qp = wl.q_positions().to(device)
    S = torch.empty((wl.batch, 1, wl.N), dtype=torch.float32, device=device)
    idx = torch.empty((wl.batch, 1, wl.k), dtype=torch.int32, device=device)
    out = torch.empty_like(q)
    nws = csa.attend_workspace_bytes(wl.batch, 1, wl.H, wl.D, wl.k + wl.W)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=device)
    q4 = torch.empty((wl.batch, 1, wl.H_I, wl.d_I // 2), dtype=torch.uint8, device=device)
    q4s = torch.empty((wl.batch, 1, wl.H_I, wl.d_I // 16), dtype=torch.uint8, device=device)

    KC = 4 * wl.k  # FP4 over-selection before the bf16 re-ranking
    cand = torch.empty((wl.batch, 1, KC), dtype=torch.int32, device=device)
    rws = torch.empty(csa.rescore_workspace_bytes(wl.batch, 1, KC, wl.k, wl.d_I), dtype=torch.uint8, device=device)

    def step(mark):
        csa.csa_quantize_fp4(qI, packed=q4, scales=q4s)
        csa.csa_index_fp4(q4, q4s, w, k4, k4s, qp, wl.m, scores=S)
        mark(0)
        csa.csa_topk(S, qp, wl.m, wl.k, idx=idx)
        mark(1)
        csa.csa_attend(q, C, idx, win, qp, wl.W, wl.scale, wl.eps, out=out, workspace=ws, win_pos0=wl.T - wl.W)

    def step2(mark):  # over-select with FP4, re-rank the candidates with the bf16 index keys
        csa.csa_quantize_fp4(qI, packed=q4, scales=q4s)
        csa.csa_index_fp4(q4, q4s, w, k4, k4s, qp, wl.m, scores=S)
        mark(0)
        csa.csa_topk(S, qp, wl.m, KC, idx=cand)
        csa.csa_rescore_topk(qI, w, kI, cand, wl.k, idx=idx, workspace=rws)
        mark(1)
        csa.csa_attend(q, C, idx, win, qp, wl.W, wl.scale, wl.eps, out=out, workspace=ws, win_pos0=wl.T - wl.W)

    steps = max(2, min(args.steps, 10))
    tot, seg = Timer(device).run(step, steps, 2, marks=2)
    t = tot / steps
    tot2, seg2 = Timer(device).run(step2, steps, 2, marks=2)
    t2 = tot2 / steps
    ib = index_bytes(wl, fp4=True)
    # bf16 indexer on the same keys for the FP4 / bf16 time ratio and the recall
    S16 = csa.csa_index(qI, w, kI, qp, wl.m)
    t16, _ = Timer(device).run(lambda mark: csa.csa_index(qI, w, kI, qp, wl.m, scores=S16), steps, 1)
    idx16 = csa.csa_topk(S16, qp, wl.m, wl.k)
    csa.csa_index_fp4(q4, q4s, w, k4, k4s, qp, wl.m, scores=S)
    idx4 = csa.csa_topk(S, qp, wl.m, wl.k)
    idx4r = csa.csa_rescore_topk(qI, w, kI, csa.csa_topk(S, qp, wl.m, KC), wl.k)
    torch.cuda.synchronize()

    def recall(a):
        r = [len(set(a[b, 0].tolist()) & set(idx16[b, 0].tolist())) / wl.k for b in range(wl.batch)]
        return round(sum(r) / len(r), 4)

    return {"workload": wl.name, "queries_per_s": wl.batch / t2, "ms_per_step": round(t2 * 1e3, 4),
            "selection": "FP4 over-select %d, bf16 re-rank to %d" % (KC, wl.k),
            "recall_vs_bf16_operand_topk": recall(idx4r),
            "index_fp4": {"ms": round(seg[0] * 1e3, 4), "hbm_gbs": round(ib / seg[0] / 1e9, 1),
                          "frac": round(ib / seg[0] / 1e9 / peaks["hbm_gbs"], 4)},
            "select_ms": {"fp4_topk_%d" % wl.k: round(seg[1] * 1e3, 4),
                          "fp4_topk_%d_plus_rerank" % KC: round(seg2[1] * 1e3, 4)},
            "single_pass": {"queries_per_s": wl.batch / t, "ms_per_step": round(t * 1e3, 4),
                            "recall_vs_bf16_operand_topk": recall(idx4)},
            "fp4_over_bf16_index_speedup": round((t16 / steps) / seg[0], 3)}


# ----------------------------------------------------------------------------- reference arm (CPU oracle)
def oracle_decode_sample(wl: W.Workload, n_queries: int = 1, min_seconds: float = 0.0):
    """The oracle on n_queries decode queries of the workload (index over every
    entry, full-sort top-k, attention), repeated on the same inputs until at
    least min_seconds have passed; returns (seconds, queries, threads)."""
    import numpy as np

    import oracle
    wl1 = wl.scaled(batch=n_queries)
    kI = W.index_keys(wl1)
    qI, w = W.index_queries(wl1), W.index_weights(wl1)
    q = W.queries(wl1)
    C = W.direct_kv(wl1)
    win = W.normal_bf16((wl1.batch, wl1.W, wl1.D), 424242)
    qp = wl1.q_positions().numpy()
    bits = W.bits
    qI_b, kI_b, q_b, C_b, win_b, w_n = bits(qI), bits(kI), bits(q), bits(C), bits(win), w.numpy()
    t0 = time.perf_counter()
    done = 0
    while True:
        S = oracle.index(qI_b, w_n, kI_b, qp, wl1.m)
        idx = oracle.topk(S, qp, wl1.m, wl1.k)
        oracle.attend(q_b, C_b, idx, win_b, qp, wl1.W, wl1.scale, wl1.eps, win_pos0=wl1.T - wl1.W)
        _ = np.asarray(idx)
        done += n_queries
        dt = time.perf_counter() - t0
        if dt >= min_seconds:
            return dt, done, oracle.num_threads()


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    wl = W.CSA_DECODE
    # a step: the oracle on one decode batch (the GPU arm's step), inputs generated outside the timing
    for _ in range(max(0, min(args.warmup, 1))):
        oracle_decode_sample(wl, n_queries=wl.batch)
    total = 0.0
    threads = 1
    steps = max(1, args.steps)
    for _ in range(steps):
        dt, _, threads = oracle_decode_sample(wl, n_queries=wl.batch)
        total += dt
    value = steps * wl.batch / total
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "queries/s",
            "n_gpus": args.gpus, "steps": steps, "warmup": args.warmup, "ms_per_step": total / steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": decode_config(wl, args.gpus),
            "cpu_baseline": {"value": value, "unit": "queries/s", "cores": threads, "kind": "oracle",
                             "sample": "the %d queries of one 128K decode batch per step (index over 32768 entries "
                                       "each, full-sort top-1024, 128x512 attention over 1152 keys)" % wl.batch},
            "e2e": {"value": value, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def decode_for_profiling(csa, args, device):
    """One 128K decode state (cache built by csa_compress) and warmup + steps
    eager decode steps, for kernel profilers: a few hundred MB on the device
    and no other launches than the cache build and the steps."""
    st = decode_cache_state(csa, W.CSA_DECODE, device, 0)
    for _ in range(args.warmup + args.steps):
        decode_step(csa, st)
    torch.cuda.synchronize()
    return {"workload": "csa_decode_128k", "steps": args.warmup + args.steps, "note": "profiling run, not timed"}


def decode_config(wl: W.Workload, world: int) -> dict:
    """The headline workload as both arms name it."""
    return {"workload": wl.name, "batch_per_gpu": wl.batch, "context": wl.T, "m": wl.m, "entries": wl.N,
            "top_k": wl.k, "heads": wl.H, "head_dim": wl.D, "indexer": [wl.H_I, wl.d_I], "window": wl.W,
            "parallelism": "replicas x%d" % world, "l2": "inputs larger than L2: 6 decode states (79 MB of step inputs each) rotate, no flush",
            "cuda_graph": True}


# ----------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extra", action="store_true", help="headline workload only")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=["prefill", "hca", "fp4", "compress", "compress_dynamic", "fp8kv", "decode"],
                    help="run one workload alone and print its JSON (for profiling); 'decode' builds one 128K "
                         "decode state and runs warmup + steps eager csa_decode_step calls")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    args.warmup = max(args.warmup, 3)

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist_init(world)
    import long_context_compressed_06_b200 as csa
    csa.load()
    peaks, peak_kind = load_peaks()
    if args.only:
        run_one = {"prefill": lambda: bench_prefill(csa, args, device, peaks),
                   "hca": lambda: bench_hca(csa, args, device, peaks),
                   "fp4": lambda: bench_fp4(csa, args, device, peaks),
                   "compress": lambda: bench_compress(csa, args, device, peaks, W.HCA_DECODE),
                   "compress_dynamic": lambda: bench_compress_dynamic(csa, args, device, peaks, W.CSA_DECODE),
                   "fp8kv": lambda: bench_fp8kv_decode(csa, args, device, peaks),
                   "decode": lambda: decode_for_profiling(csa, args, device),
                   }[args.only]
        res = run_one()
        rc = csa.csa_sync_status()
        if rc != 0:
            raise RuntimeError("device status: %s" % csa.strerror(rc))
        if rank == 0:
            print(json.dumps(res))
        barrier(world)
        return 0

    head, _ = bench_csa_decode(csa, args, device, world, rank, peaks)
    rc = csa.csa_sync_status()
    if rc != 0:
        raise RuntimeError("device status after the timed steps: %s" % csa.strerror(rc))
    extra = {}
    if not args.no_extra and rank == 0:
        torch.cuda.empty_cache()
        extra["csa_prefill_64k"] = bench_prefill(csa, args, device, peaks)
        torch.cuda.empty_cache()
        extra["hca_decode_1m"] = bench_hca(csa, args, device, peaks)
        torch.cuda.empty_cache()
        extra["fp4_index_decode_1m"] = bench_fp4(csa, args, device, peaks)
        torch.cuda.empty_cache()
        extra["fp8kv_decode_128k"] = bench_fp8kv_decode(csa, args, device, peaks)
        torch.cuda.empty_cache()
        extra["compress_m4_128k"] = bench_compress(csa, args, device, peaks, W.CSA_DECODE)
        extra["compress_m128_1m"] = bench_compress(csa, args, device, peaks, W.HCA_DECODE)
        torch.cuda.empty_cache()
        extra["compress_dynamic_m4_128k"] = bench_compress_dynamic(csa, args, device, peaks, W.CSA_DECODE)
        extra["compress_dynamic_m128_1m"] = bench_compress_dynamic(csa, args, device, peaks, W.HCA_DECODE)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        wl = W.CSA_DECODE
        dt, nq_done, threads = oracle_decode_sample(wl, n_queries=wl.batch, min_seconds=10.0)
        cpu = {"value": nq_done / dt, "unit": "queries/s", "cores": threads, "kind": "oracle",
               "sample": "the %d queries of one 128K decode batch (index over 32768 entries each, full-sort "
                         "top-1024, 128x512 attention over 1152 keys), %d times on the same inputs: %d queries "
                         "in %.1f s" % (wl.batch, nq_done // wl.batch, nq_done, dt)}
    rc = csa.csa_sync_status()
    if rc != 0:
        raise RuntimeError("device status: %s" % csa.strerror(rc))
    if rank == 0:
        wl = W.CSA_DECODE
        head["roofline"]["peak_source"] = peak_kind + " (burst, kernel timed alone)"
        line = {"metric": METRIC,
                "value": head["value"], "unit": "queries/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": decode_config(wl, world),
                "roofline": head["roofline"], "step": head["step"], "cpu_baseline": cpu, "e2e": head["e2e"],
                "gpu_launches": head["launches"], "clocks": head["clocks"], "workloads": extra}
        print(json.dumps(line))
    barrier(world)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
