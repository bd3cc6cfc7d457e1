#!/usr/bin/env python
"""Benchmark of the MS-GLA layer forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one MS-GLA layer forward over one batch of the 340M-shaped layer
(B=8, L=2048, d=1024, scales {1,2,4} with heads [2,1,1], d_k=256, d_v=512) on
seeded synthetic inputs (see scale_gated_linear_b200/workloads.py). With N > 1
(one process per GPU under torch.distributed.run) every rank runs its own batch
of 8 sequences: batch sequences are independent, so the work is sharded by
sequence with no collective on the data path ("scaling": "weak").

Variants of the same step: --mask left|right|random times the masked forward
(valid-token mask in the pooling, Eq. (8); e2e is then not measured: the host
entry point takes no mask) and --head-norm enables the optional per-head RMS
norm of the GLA output.

Prints one JSON line on rank 0. Timing: W untimed warm-up steps, then K timed
steps, each bracketed by CUDA events on the launching stream with a 256 MiB
write between steps to flush the 126 MB L2, followed by a 256 MiB read so that
the step does not pay for writing back the flush's own dirty lines. The kernels
of a forward are
launched so that each may start while the previous one finishes, and an event
between two kernels takes that overlap away, so the timed steps record events
only at the step boundaries, and every fourth timed step also around the
dominant kernel (for the roofline: its mean over those steps); the dominant
kernel and the per-kernel table (kernel_ms) come from separate forwards with an
event at every kernel boundary. The line also carries the
forward's workspace bytes (`memory`) and, beside the single-scale GLA layer's
throughput, its workspace bytes and the ratio of the two.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MS-GLA layer fwd tokens/sec @d=1024,L=2048"
UNIT = "tokens/s"
WORKLOAD = "msgla_340m"
SINGLE_SCALE_WORKLOAD = "gla_340m"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


# --------------------------------------------------------------------- helpers
def shard_rows(global_rows: int, rank: int, world: int) -> range:
    """Contiguous block of batch rows owned by `rank` (weak scaling gives every rank
    the same count; any remainder goes to the lowest ranks)."""
    base, rem = divmod(global_rows, world)
    start = rank * base + min(rank, rem)
    return range(start, start + base + (1 if rank < rem else 0))


def max_over_ranks(value: float, world: int, device=None) -> float:
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def algorithmic_counts(w, B: int, L: int) -> dict:
    """Algorithmic FLOPs (tensor work) and bytes per kernel of one forward.

    FLOPs count only what the layer computes, per branch at pooled length: the
    q/k/v projections 2d(2 d_k + d_v) per head, the gate's two low-rank factors
    2 d r + 2 r h d_k, the chunkwise GLA 4 d_k d_v + C (d_k + d_v) per head with
    C the workload's configured chunk (the causal half of the intra-chunk
    products), the output projection 2 d_v d per head, plus the fusion logits
    2 d |S| and 6 d of elementwise work per token; bytes count each kernel's
    compulsory global-memory traffic."""
    C = w.chunk
    r = w.gate_rank
    nS = len(w.scales)
    out = {}
    rows = {s: B * math.ceil(L / s) for s in w.scales}
    # gate inputs by linearity from the unpooled rows (each branch's W_g1 and
    # W_fuse) and the pooled rows: one pass over X (pool_u), or a GEMM and a
    # pooling kernel for scale sets the fused kernel does not take
    u_flops = sum(rows[s] * 2 * w.d * r for s in w.scales) + B * L * 2 * w.d * nS
    u_bytes = B * L * (16 + nS * -(-r // 16) * 16) * 4
    pooled = sum(rows[s] * w.d * 2 for s in w.scales if s > 1)
    if all(s in (1, 2, 4, 8) for s in w.scales) and 16 + nS * -(-r // 16) * 16 <= 256:
        out["pool_u"] = {"flops": u_flops, "bytes": B * L * w.d * 2 + u_bytes + pooled}
    else:
        out["gate_inputs"] = {"flops": u_flops, "bytes": B * L * w.d * 2 + u_bytes}
        if pooled:
            out["pool"] = {"bytes": B * L * w.d * 2 + pooled}
    # gate exponents (fp32) and chunk decays written once
    out["gate"] = {"bytes": sum(rows[s] * h * w.d_k * 4 + 2 * B * math.ceil(rows[s] / B / 128) * h * w.d_k * 4
                                for s, h in zip(w.scales, w.heads))}
    out["proj_gemm"] = {"flops": sum(rows[s] * 2 * h * (w.d * (2 * w.d_k + w.d_v) + r * w.d_k)
                                     for s, h in zip(w.scales, w.heads))}
    out["gla"] = {"flops": sum(rows[s] * h * (4 * w.d_k * w.d_v + C * (w.d_k + w.d_v))
                               for s, h in zip(w.scales, w.heads))}
    coarse = [(s, h) for s, h in zip(w.scales, w.heads) if s != 1]
    if coarse:
        out["out_gemm_coarse"] = {"flops": sum(rows[s] * 2 * h * w.d_v * w.d for s, h in coarse)}
    if 1 in w.scales:
        h1 = dict(zip(w.scales, w.heads))[1]
        out["out_gemm_fused"] = {"flops": rows[1] * 2 * h1 * w.d_v * w.d}
    else:  # the hold and fusion as a memory pass: held rows and weights in, O out
        out["hold_fuse"] = {"bytes": sum(rows[s] * w.d * 2 for s in w.scales) + B * L * nS * 4 + B * L * w.d * 2}
    if getattr(w, "head_norm", False):  # read + write of the GLA output, in place
        out["head_norm"] = {"bytes": sum(rows[s] * h * w.d_v * 2 * 2 for s, h in zip(w.scales, w.heads))}
    total_flops = sum(v.get("flops", 0) for v in out.values()) + B * L * 6 * w.d
    weights = sum(h * (2 * w.d_k + w.d_v) * w.d * 2 + r * w.d * 2 + h * w.d_k * r * 4 + w.d * h * w.d_v * 2
                  for s, h in zip(w.scales, w.heads))
    layer_bytes = 2 * B * L * w.d * 2 + weights
    return {"kernels": out, "total_flops": total_flops, "layer_bytes": layer_bytes}


# source files that decide what each timed kernel does (its own file and the shared headers)
KERNEL_SOURCES = {
    "proj_gemm": "k_gemm.cu", "out_gemm_coarse": "k_gemm.cu", "out_gemm_fused": "k_gemm.cu",
    "gla": "k_gla.cu", "gla_state": "k_gla.cu", "gla_scan": "k_gla.cu",
    "gate_inputs": "k_gemm.cu", "pool": "k_aux.cu", "gate": "k_aux.cu", "pool_u": "k_pool.cu", "head_norm": "k_aux.cu", "hold_fuse": "k_aux.cu",
}


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "scale_gated_linear_b200", "csrc")
    for name in (KERNEL_SOURCES[kernel], "msgla_internal.h", "sm100_ptx.cuh"):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, workload: str):
    """Per-launch DRAM bytes (read + write) of `kernel` from the committed ncu
    summary, or None if there is none or the kernel's sources changed since."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    e = t.get("kernels", {}).get(workload, {}).get(kernel)
    if not e or e.get("source_hash") != kernel_source_hash(kernel):
        return None
    return e.get("dram_bytes")


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""

    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.rows = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == 9 and (self.uuid is None or self.uuid in parts[0]):
                self.rows.append(parts)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows)}


def numpy_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(w, inp, rows_budget_s: float, prefix: int | None = None, mask=None):
    """Run the fp64 oracle on whole batch rows (or a prefix of them) until about
    `rows_budget_s` seconds have passed. Returns (tokens, seconds, description)."""
    import numpy as np

    import oracle
    from scale_gated_linear_b200 import workloads as wl
    f = wl.to_float64(inp)
    L = f["X"].shape[1] if prefix is None else prefix
    done, t0 = 0, time.perf_counter()
    for b in range(f["X"].shape[0]):
        oracle.layer_forward(f["X"][b:b + 1, :L], f, w.scales, w.heads, w.d_k, w.d_v,
                             gate_normalizer=w.gate_normalizer,
                             mask=None if mask is None else mask[b:b + 1, :L].numpy(),
                             head_norm_eps=w.norm_eps if w.head_norm else None)
        done += 1
        if time.perf_counter() - t0 >= rows_budget_s:
            break
    dt = time.perf_counter() - t0
    desc = f"{done} batch row(s) x {L} positions of {w.name} (B={w.B}, L={w.L}), fp64 oracle, numpy"
    return done * L, dt, desc


# --------------------------------------------------------------------- reference arm
def run_reference(args) -> int:
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from scale_gated_linear_b200 import workloads as wl
    w = wl.WORKLOADS[args.workload]
    inp = wl.make_inputs(w, B=1)
    prefix = min(w.L, args.ref_prefix)
    times = []
    for k in range(args.warmup + args.steps):
        tok, dt, desc = oracle_sample(w, inp, 0.0, prefix=prefix)
        if k >= args.warmup:
            times.append(dt)
    total = sum(times)
    value = len(times) * prefix / total
    cores = numpy_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{w.name}: one sequence prefix of {prefix} of B={w.B} x L={w.L}, d={w.d}, "
                               f"scales {list(w.scales)} heads {list(w.heads)}, d_k={w.d_k}, d_v={w.d_v}",
                   "l2": "n/a (CPU)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"each step: first {prefix} positions of one batch row (fp64 numpy oracle)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------- decode
def decode_bytes(w, B: int, t: int) -> int:
    """Algorithmic HBM bytes of the decode step at position t: packed weights of
    the branches that step (projection rows and W_o, 2 bytes each), their fp32
    state read and written, every coarse branch's block sum read and written and
    latest output read, the token in and the output out."""
    dkp = 128 if w.d_k <= 128 else 256
    dvp = -(-w.d_v // 128) * 128
    rp = -(-w.gate_rank // 16) * 16
    n = 2 * B * w.d * 2 + len(w.scales) * w.d * 2  # x, O, W_fuse
    for s, h in zip(w.scales, w.heads):
        if s > 1:
            n += B * w.d * (4 + 4 + 2)
        if (t + 1) % s == 0:
            n += (h * (2 * dkp + dvp) + rp) * w.d * 2 + w.d * h * dvp * 2
            n += 2 * B * h * dkp * dvp * 4
    return n


def run_decode(args) -> int:
    import torch

    from scale_gated_linear_b200 import MSGLA
    from scale_gated_linear_b200 import workloads as wl
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1 and rank > 0:  # decode is measured on one GPU (independent replicas otherwise)
        return 0
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = wl.WORKLOADS[args.workload]
    if args.batch:
        w = w.replace(B=args.batch)
    if args.head_norm:
        w = w.replace(head_norm=True)
    period = 1
    for s in w.scales:
        period = period * s // math.gcd(period, s)
    inp = wl.make_inputs(w, L=period)
    layer = MSGLA.from_workload(w, inp, device=local)
    X = inp["X"].to(dev)
    B = w.B
    cache = layer.new_cache(B)
    ws = torch.empty(max(layer.step_workspace_size(B), 1), dtype=torch.uint8, device=dev)
    out = torch.empty(B, w.d, dtype=torch.bfloat16, device=dev)
    xs = [X[:, i].contiguous() for i in range(period)]
    flush_buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    t = 0

    def cycle(st=stream):
        nonlocal t
        for i in range(period):
            layer.step(xs[i], t, cache, out=out, workspace=ws, stream=st)
            t += 1

    for _ in range(args.warmup):
        flush_buf.fill_(1)
        cycle()
    torch.cuda.synchronize()
    layer.check_status()
    graph = None
    if args.graph:
        # which branches step depends only on t mod period: one captured cycle
        # replays every later cycle (the tokens are read from the fixed buffers xs)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            cycle(torch.cuda.current_stream())
        torch.cuda.synchronize()
        for _ in range(2):
            graph.replay()
        torch.cuda.synchronize()
        layer.check_status()
    sampler = ClockSampler(None)
    sampler.start()
    time.sleep(0.3)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_first = t
    for k in range(args.steps):
        flush_buf.fill_(1)
        ev[k][0].record(stream)
        if graph is not None:
            graph.replay()
            t += period
        else:
            cycle()
        ev[k][1].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    layer.check_status()
    total_ms = sum(a.elapsed_time(b) for a, b in ev)
    tokens = B * period * args.steps
    nbytes = sum(decode_bytes(w, B, tt) for tt in range(t_first, t_first + period))
    cyc_ms = total_ms / args.steps
    peaks, peak_kind = load_peaks()
    achieved = nbytes / (cyc_ms * 1e-3) / 1e9
    line = {
        "metric": "MS-GLA decode tokens/sec (one token per sequence per step)", "value": tokens / (total_ms / 1e3),
        "unit": UNIT, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": cyc_ms, "tokens_per_step": B * period, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32 state, f16/bf16 tensor-core operands; bf16 in/out", "data": "synthetic",
        "config": {"workload": f"{w.name}: decode of B={B} sequences, one step = {period} tokens (every branch "
                               f"steps once), d={w.d}, scales {list(w.scales)} heads {list(w.heads)}, "
                               f"d_k={w.d_k}, d_v={w.d_v}", "l2": "flushed between timed steps (256 MiB write)"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "kernel": "whole decode step",
                     "bytes_per_step": nbytes, "peak_source": peak_kind},
        "us_per_token_position": 1e3 * cyc_ms / period,
        "launch": "one CUDA graph per step (captured cycle)" if graph is not None else "eager msgla_step calls",
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    del graph
    layer.close()
    return 0


# --------------------------------------------------------------------- our arm
def profile_kernels(layer, X, O, ws, names, reps: int, flush, mask=None) -> dict:
    """Per-kernel durations (ms) from `reps` forwards with an event at every
    kernel boundary (each event keeps the next kernel from starting early, so
    these intervals add up to a little more than an untouched step)."""
    import torch
    stream = torch.cuda.current_stream()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(reps)]
    for k in range(reps):
        flush()
        layer.forward_profiled(X, O, ws, ev[k], stream, mask=mask)
    torch.cuda.synchronize()
    return {n: statistics.mean(ev[k][i].elapsed_time(ev[k][i + 1]) for k in range(reps)) for i, n in enumerate(names)}


def run_ours(args) -> int:
    import torch
    import torch.distributed as dist

    from scale_gated_linear_b200 import MSGLA
    from scale_gated_linear_b200 import workloads as wl

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    w = wl.WORKLOADS[args.workload]
    if args.batch:
        w = w.replace(B=args.batch)
    if args.head_norm:
        w = w.replace(head_norm=True)
    peaks, peak_kind = load_peaks()
    cpu_line = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        inp0 = wl.make_inputs(w, B=min(w.B, 4))
        m0 = None if args.mask == "none" else wl.make_mask(min(w.B, 4), w.L, args.mask, seed=w.seed)
        tok, dt, desc = oracle_sample(w, inp0, args.cpu_seconds, mask=m0)
        cpu_line = {"value": tok / dt, "unit": UNIT, "cores": numpy_threads(), "kind": "oracle", "sample": desc}

    def measure(wk, steps, warmup, e2e: bool, mask_kind: str = "none"):
        inp = wl.make_inputs(wk)
        if rank > 0:  # this rank's own batch of sequences (same weights)
            g = torch.Generator().manual_seed(wk.seed * 1000 + rank)
            X = torch.randn(wk.B, wk.L, wk.d, generator=g)
            inp["X"] = (X / X.pow(2).mean(-1, keepdim=True).sqrt()).to(torch.bfloat16)
        layer = MSGLA.from_workload(wk, inp, device=local)
        X = inp["X"].to(dev)
        M = None if mask_kind == "none" else wl.make_mask(wk.B, wk.L, mask_kind, seed=wk.seed + rank).to(dev)
        O = torch.empty_like(X)
        ws = layer.alloc_workspace(wk.B, wk.L)
        # L2 flush between steps: a 256 MiB write, then a 256 MiB read that evicts the
        # write's dirty lines, so every timed step starts from a cold L2 that holds
        # neither its inputs nor write-backs owed by the flush itself
        flush_buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
        flush_rd = torch.ones(256 * 1024 * 1024 // 8, dtype=torch.int64, device=dev)
        flush = lambda: (flush_buf.fill_(1), flush_rd.sum())
        names = layer.launch_names(wk.B, wk.L)
        n_ev = len(names) + 1
        stream = torch.cuda.current_stream()
        # warm-up steps, then the dominant kernel from a profiled pass
        for _ in range(warmup):
            flush()
            layer.forward(X, out=O, workspace=ws, stream=stream, mask=M)
        prof = profile_kernels(layer, X, O, ws, names, max(3, warmup), flush, mask=M)
        # the longest kernel with an algorithmic count (the segment scan and state
        # pass of long sequences have none)
        counted = algorithmic_counts(wk, wk.B, wk.L)["kernels"]
        dom = max((k for k in prof if k in counted), key=prof.get)
        i_dom = names.index(dom)
        # Timed steps record the step boundaries; every fourth one (the last one when
        # there are fewer than four) also records the dominant kernel's boundaries.
        # An event between two kernels keeps the second from starting before the
        # first has finished (it breaks the programmatic dependent launch and the
        # GLA's per-chunk start), which costs about 10 us per step at msgla_340m,
        # so only the sampled steps pay it; the value still counts every step.
        sampled = [k for k in range(steps) if k % 4 == 3] or [steps - 1]
        ev = [[torch.cuda.Event(enable_timing=True)
               if i in (0, n_ev - 1) or (k in sampled and i in (i_dom, i_dom + 1)) else None
               for i in range(n_ev)] for k in range(steps)]
        torch.cuda.synchronize()
        layer.check_status()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        sampler = ClockSampler(getattr(torch.cuda.get_device_properties(dev), "uuid", None)
                               and str(torch.cuda.get_device_properties(dev).uuid))
        sampler.start()
        time.sleep(0.3)
        launches = 0
        for k in range(steps):
            flush()
            launches += layer.forward_profiled(X, O, ws, ev[k], stream, mask=M)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        clocks = sampler.stop()
        layer.check_status()
        step_ms = [ev[k][0].elapsed_time(ev[k][-1]) for k in range(steps)]
        dom_ms = [ev[k][i_dom].elapsed_time(ev[k][i_dom + 1]) for k in sampled]
        total_ms = max_over_ranks(sum(step_ms), world, dev)
        res = {"total_ms": total_ms, "step_ms": step_ms, "dominant": dom, "dominant_ms": dom_ms,
               "profiled_ms": prof, "launches": launches, "clocks": clocks, "tokens_per_step": wk.B * wk.L,
               "workspace_bytes": int(ws.numel())}
        if e2e:
            wsh = layer.alloc_workspace(wk.B, wk.L, host_staging=True)
            Xh = inp["X"].pin_memory()
            Oh = torch.empty_like(Xh).pin_memory()
            for _ in range(max(1, warmup)):
                layer.forward_host(Xh, Oh, wsh)
            e_ms = []
            for _ in range(steps):
                flush()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                layer.forward_host(Xh, Oh, wsh, stream)
                b.record(stream)
                b.synchronize()
                e_ms.append(a.elapsed_time(b))
            res["e2e_ms"] = max_over_ranks(sum(e_ms), world, dev)
            res["io_bytes"] = Xh.numel() * 2
            del wsh
        layer.close()
        del ws, flush_buf, flush_rd
        torch.cuda.empty_cache()
        return res

    r = measure(w, args.steps, args.warmup, e2e=not args.no_e2e and args.mask == "none", mask_kind=args.mask)
    tokens = r["tokens_per_step"] * args.steps * world
    value = tokens / (r["total_ms"] / 1e3)
    counts = algorithmic_counts(w, w.B, w.L)
    dominant = r["dominant"]
    dom_ms = statistics.mean(r["dominant_ms"])
    kc = counts["kernels"][dominant]
    if "flops" in kc and dominant not in ("gate_inputs", "pool_u"):
        achieved = kc["flops"] / (dom_ms * 1e-3) / 1e12
        peak = peaks["bf16_tflops"]
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak}
    else:
        achieved = kc["bytes"] / (dom_ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak}
    roof.update({"kernel": dominant, "scope": "dominant kernel only (the whole layer: path_roofline)",
                 "peak_source": f"{peak_kind} (MEASURED_PEAKS.json burst)"
                 if peak_kind == "measured" else "fallback", "traffic": traffic_for(dominant, f"{w.name}/B{w.B}/L{w.L}")
                 if args.mask == "none" and not w.head_norm else None,
                 "kernel_ms": dom_ms})
    step_ms = r["total_ms"] / args.steps
    path_tf = counts["total_flops"] / (step_ms * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16/bf16 tensor-core operands, f32 accumulate; bf16 in/out",
        "data": "synthetic (seeded N(0,1) rows RMS-normalised, weights N(0,0.02))",
        "config": {"workload": f"{w.name}: B={w.B} per GPU, L={w.L}, d={w.d}, scales {list(w.scales)} heads "
                               f"{list(w.heads)}, d_k={w.d_k}, d_v={w.d_v}, gate rank {w.gate_rank}, chunk {w.chunk} "
                               f"(kernel chunk 128)"
                               + (f", {args.mask}-padding mask" if args.mask != "none" else "")
                               + (", head RMS norm" if w.head_norm else ""),
                   "global_batch": w.B * world, "seq_len": w.L, "parallelism": f"sequence-sharded x{world}",
                   "l2": "flushed between timed steps (256 MiB write, then a 256 MiB read: cold and clean)"},
        "roofline": roof,
        "path_roofline": {"scope": "whole layer forward (the >= 50 % target)", "bound": "tensor",
                          "achieved": path_tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                          "frac": path_tf / peaks["bf16_tflops"], "flops_per_step": counts["total_flops"],
                          "chunk_in_count": w.chunk},
        "kernel_ms": r["profiled_ms"],
        "kernel_ms_note": "separate forwards with an event at every kernel boundary (which keeps each kernel "
                          "from starting before the previous one ends); the timed steps record only the step "
                          "boundaries, and every fourth one also the dominant kernel's (the roofline's "
                          "kernel_ms is their mean)",
        "gpu_launches": r["launches"],
        "clocks": r["clocks"],
        "memory": {"workspace_bytes": r["workspace_bytes"],
                   "note": "device intermediates of one forward (the caller-owned workspace)"},
    }
    if "e2e_ms" in r:
        line["e2e"] = {"value": tokens / (r["e2e_ms"] / 1e3), "unit": UNIT,
                       "h2d_bytes_per_step": r["io_bytes"], "d2h_bytes_per_step": r["io_bytes"]}
    elif args.mask != "none":
        line["e2e"] = {"value": None, "unit": UNIT, "note": "not measured: the host-buffer entry point takes no mask"}
    if world == 1 and not args.no_gla_baseline and args.mask == "none" and not w.head_norm:
        g = measure(wl.WORKLOADS[SINGLE_SCALE_WORKLOAD], max(3, args.steps // 2), args.warmup, e2e=False)
        g_ms = g["total_ms"] / max(3, args.steps // 2)
        line["gla_baseline"] = {"workload": SINGLE_SCALE_WORKLOAD, "value": g["tokens_per_step"] / (g_ms * 1e-3),
                                "unit": UNIT, "ms_per_step": g_ms, "time_ratio_msgla_over_gla": step_ms / g_ms,
                                "workspace_bytes": g["workspace_bytes"],
                                "workspace_ratio_msgla_over_gla": r["workspace_bytes"] / g["workspace_bytes"]}
    if cpu_line is not None:
        line["cpu_baseline"] = cpu_line
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-gla-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="budget of the CPU oracle baseline")
    ap.add_argument("--ref-prefix", type=int, default=512, help="positions per reference-arm step")
    ap.add_argument("--mask", choices=("none", "left", "right", "random"), default="none",
                    help="time the masked forward with this valid-token mask")
    ap.add_argument("--head-norm", action="store_true", help="enable the per-head RMS norm of the GLA output")
    ap.add_argument("--batch", type=int, default=0, help="sequences per GPU (default: the workload's)")
    ap.add_argument("--graph", action="store_true", help="with --decode: replay one captured step as a CUDA graph")
    ap.add_argument("--decode", action="store_true",
                    help="time token-by-token decode (msgla_step) instead of the whole-sequence forward")
    args = ap.parse_args(argv)
    if args.decode:
        return run_decode(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
