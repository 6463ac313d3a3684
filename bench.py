#!/usr/bin/env python
"""Benchmark of the CoWA hot path on B200.

One step = one pass of the whole path over one batch of synthetic inputs:
cowa_fwd (schedule + forward), cowa_bwd (schedules, delta, dK/dV pass, dQ
pass) and cowa_decode of one new token per sequence against the same K/V as
its cache (split-KV + merge).  The default workload is the 128K training
operator (B=1, L=131072, Hq=32, Hkv=8, d=128, quad (128, 8192, 0, 15360)),
the largest configuration that fits one GPU; ``--workload recall8k`` or
``llm14b_32k`` selects a smaller one.

Metric: effective TFLOP/s counted on visible pairs only -- 4*d flops per
pair forward, 10*d backward, 4*d per visible key and query head in decode --
over the step time; decode GB/s on visible K+V bytes is reported beside it.
Timing: CUDA events on the launching stream, L2 flushed (a 512 MiB write)
before every timed step, max over ranks.  Multi-GPU, no collective on the
data path in either mode: by default every rank runs its own batch
(data-parallel replicas, weak scaling); with ``--parallel heads`` rank r
takes KV heads [r*Hkv/N, (r+1)*Hkv/N) of the one workload with their query
heads and passes the first one's global index as kv_head_offset (KV-head
tensor parallelism, strong scaling).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--parallel dp|heads]
  python bench.py --impl reference ...   # the fp64 CPU oracle, timed on host cores
"""
import argparse
import dataclasses
import datetime
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# Query rows of the oracle's bounded samples (batch 0, the last rows of the
# sequence): the CPU-baseline leg, about 10-20 s of fp64 work on 16 host
# cores, and one reference-arm step, a few seconds, so that 25 of them end
# within minutes.  The oracle's cost is linear in the rows (each row of the
# 128K operator takes about 0.14 s of 16 cores, forward + backward).
CPU_ROWS = {"tiny": 512, "recall8k": 4096, "llm14b_32k": 512, "op128k": 96}
REF_ROWS = {"tiny": 512, "recall8k": 512, "llm14b_32k": 64, "op128k": 16}

# A kernel timed inside a step this long, with the timed steps back to back
# for seconds, runs under the power cap like the sustained GEMM loop of the
# peak measurement, so its fraction is taken of the sustained bf16 figure;
# shorter steps use the burst figure.
LONG_STEP_MS = 20.0


# --------------------------------------------------------------- counting ----
def row_visible_counts(Lq, Lk, quad, h):
    """Visible keys of every query row of KV head h (int64 [Lq]): the size of
    the union of the sink, near and long key intervals of the row."""
    S, N, G, W = (int(x) for x in quad)
    p = np.arange(Lq, dtype=np.int64) + (Lk - Lq)
    c = N + G + h * W
    e = c + W
    zero = np.zeros_like(p)
    ivs = [
        (zero, np.minimum(S, p + 1)),                          # sink  [0, S)
        (np.maximum(0, p - N + 1), p + 1 if N > 0 else zero),  # near  (p-N, p]
        (np.maximum(0, p - e + 1), np.maximum(0, p - c + 1) if W > 0 else zero),  # long
    ]
    lo = np.stack([np.where(a < b, a, 0) for a, b in ivs], axis=1)
    hi = np.stack([np.where(a < b, b, 0) for a, b in ivs], axis=1)
    hi = np.where(p[:, None] >= 0, hi, 0)
    lo = np.where(hi > lo, lo, 0)
    hi = np.where(hi > lo, hi, 0)
    order = np.argsort(lo + (hi == 0) * (1 << 40), axis=1, kind="stable")
    lo = np.take_along_axis(lo, order, axis=1)
    hi = np.take_along_axis(hi, order, axis=1)
    total = np.zeros_like(p)
    reach = np.zeros_like(p)  # end of the union so far
    for a in range(3):
        start = np.maximum(lo[:, a], reach)
        total += np.maximum(0, hi[:, a] - start)
        reach = np.maximum(reach, hi[:, a])
    return total


def visible_pairs(B, Lq, Lk, Hq, Hkv, quad, kv_head_offset=0, rows=None):
    """Visible (query, key) pairs over all batches and query heads."""
    g = Hq // Hkv
    tot = 0
    for h in range(Hkv):
        cnt = row_visible_counts(Lq, Lk, quad, h + kv_head_offset)
        if rows is not None:
            cnt = cnt[rows]
        tot += int(cnt.sum()) * g
    return tot * B


def decode_visible_keys(seqlens, Hkv, quad, kv_head_offset=0):
    """Visible keys summed over sequences and KV heads for one decode step."""
    tot = 0
    for L in seqlens:
        for h in range(Hkv):
            tot += int(row_visible_counts(1, int(L), quad, h + kv_head_offset)[0]) if L > 0 else 0
    return tot


def max_over_ranks(values, world, device):
    """Element-wise max of a list of floats over all ranks (the slowest rank
    sets the time of a step)."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def sum_over_ranks(values, world, device):
    """Element-wise sum of a list of numbers over all ranks (whole-job work)."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return [float(x) for x in t.cpu()]


def h0_mode(args, world):
    """True when the run shards KV heads over more than one GPU."""
    return args.parallel == "heads" and world > 1


def head_shard(wl, rank, world, parallel):
    """The rank's part of a workload and its first global KV head.  Replicas
    ("dp") run all of it; KV-head sharding ("heads") gives rank r the KV heads
    [r*Hkv/R, (r+1)*Hkv/R) and their g query heads each (contiguous GQA
    groups), so its windows stay those of its global heads."""
    if parallel == "dp" or world == 1:
        return wl, 0
    if wl.Hkv % world:
        raise SystemExit("--parallel heads: %s has %d KV heads, not divisible by %d GPUs"
                         % (wl.name, wl.Hkv, world))
    per = wl.Hkv // world
    return dataclasses.replace(wl, Hq=wl.Hq // world, Hkv=per), rank * per


# ----------------------------------------------------------------- clocks ----
class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        time.sleep(0.25)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, smax, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = max(smax, float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ peaks ----
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# Source files each kernel is built from: its traffic record is valid only
# while their hash matches the one stored beside the counters.
KERNEL_SOURCES = {
    "fwd_sm100": ["fwd_sm100.cu"],
    "dkdv_sm100": ["bwd_sm100.cu"],
    "dq_sm100": ["bwd_sm100.cu"],
    "bwd_prep": ["bwd_sm100.cu"],
    "decode_split": ["decode.cu"],
    "decode_combine": ["decode.cu"],
    "mala_fwd": ["mala.cu", "mala_d128.cu"],
    "varlen_worklist": ["worklist.cu"],
}
SHARED_SOURCES = ["common.cuh", "kernels.cuh", "sm100.cuh"]


def strip_comments(src):
    """C/C++ source without its comments and blank lines, trailing spaces
    removed: what the compiler sees of it, so that editing a comment does not
    mark a kernel as changed.  String and character literals are kept whole."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            out.append(" ")
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = (ln.rstrip() for ln in "".join(out).splitlines())
    return "\n".join(ln for ln in lines if ln) + "\n"


def kernel_source_sha(kernel):
    """First 16 hex digits of sha256 over the code (comments stripped) of the
    kernel's source files."""
    import hashlib
    csrc = os.path.join(ROOT, "structured_sparse_attention_block_b200", "csrc")
    h = hashlib.sha256()
    for name in sorted(KERNEL_SOURCES.get(kernel, []) + SHARED_SOURCES):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode() + b"\0" + strip_comments(f.read()).encode())
    return h.hexdigest()[:16]


def load_traffic(kernel, workload):
    """DRAM bytes (read + write) per launch from the committed ncu counters,
    or None when none were taken on the kernel's current sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            entries = json.load(f)
    except (OSError, ValueError):
        return None
    if kernel not in KERNEL_SOURCES:
        return None
    digest = kernel_source_sha(kernel)
    for e in entries:
        if e.get("kernel") == kernel and e.get("workload") == workload and e.get("src_sha") == digest:
            return e.get("bytes_per_launch")
    return None


def kernel_work(wl, pairs, dec_keys):
    """Algorithmic work of one launch of each library kernel on a workload:
    (bound, amount, unit of amount, how it is counted).  Tensor-bound kernels
    count 2*d flops per visible (query head, key) pair and GEMM; HBM-bound
    ones the bytes they must move once."""
    d, B, Lq, Hq, Hkv = wl.d, wl.B, wl.Lq, wl.Hq, wl.Hkv
    g = Hq // Hkv
    rows = B * Hq * Lq
    lq_pad = -(-Lq // 64) * 64
    return {
        "fwd_sm100": ("tensor", pairs * 4 * d, "flop",
                      "4*d flops per visible pair (S = QK^T, O += PV), %d pairs" % pairs),
        "dkdv_sm100": ("tensor", pairs * 8 * d, "flop",
                       "8*d flops per visible pair (S^T, dP^T, dV += P^T dO, dK += dS^T Q), %d pairs" % pairs),
        "dq_sm100": ("tensor", pairs * 6 * d, "flop",
                     "6*d flops per visible pair (S, dP, dQ += dS K), %d pairs" % pairs),
        "bwd_prep": ("hbm", rows * (2 * d * 2 + 4) + B * Hq * lq_pad * 8, "byte",
                     "read O and dO (bf16) and LSE, write 8 bytes per padded row"),
        "decode_split": ("hbm", dec_keys * 2 * d * 2, "byte",
                         "visible K and V bytes, %d visible (KV head, key) pairs" % dec_keys),
    }


# ------------------------------------------------------------- GPU arm ----
def run_cowa(args, rank, world, local_rank):
    import torch.distributed as dist

    import structured_sparse_attention_block_b200 as cowa
    from structured_sparse_attention_block_b200.inputs import WORKLOADS, training_inputs

    wl_job = WORKLOADS[args.workload]
    if wl_job.kind != "train":
        raise SystemExit("the step workload must be a training workload")
    wl, h0 = head_shard(wl_job, rank, world, args.parallel)
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    q, k, v, do = training_inputs(wl.B, wl.Lq, wl.Lk, wl.Hq, wl.Hkv, wl.d, device=dev, seed=1000 * rank)
    quad = wl.quad
    # decode: the last query row of every sequence against its full K/V as cache
    qd = q[:, -1:].contiguous()
    seqlens = torch.full((wl.B,), wl.Lk, dtype=torch.int32, device=dev)

    o = torch.empty_like(q)
    lse = torch.empty((wl.B, wl.Hq, wl.Lq), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    od = torch.empty_like(qd)
    lsed = torch.empty((wl.B, wl.Hq), dtype=torch.float32, device=dev)
    ws_f = torch.empty(cowa.cowa_fwd_workspace_size(q, k, quad, h0), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(cowa.cowa_bwd_workspace_size(q, k, quad, h0), dtype=torch.uint8, device=dev)
    ws_d = torch.empty(cowa.cowa_decode_workspace_size(qd, k, quad, h0), dtype=torch.uint8, device=dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        cowa.cowa_fwd(q, k, v, quad, kv_head_offset=h0, out=o, lse=lse, workspace=ws_f)
        if ev is not None:
            ev[1].record(stream)
        cowa.cowa_bwd(q, k, v, o, lse, do, quad, kv_head_offset=h0, dq=dq, dk=dk, dv=dv, workspace=ws_b)
        if ev is not None:
            ev[2].record(stream)
        cowa.cowa_decode(qd, k, v, seqlens, quad, kv_head_offset=h0, out=od, lse=lsed, workspace=ws_d)
        if ev is not None:
            ev[3].record(stream)

    # warm-up; all but the first step are traced kernel by kernel, which
    # names the kernel with the largest share of the step
    for i in range(args.warmup):
        if i == 1:
            cowa.cowa_trace_start(32 * args.warmup + 64)
        flush.zero_()
        step()
    torch.cuda.synchronize()
    cowa.cowa_trace_stop()
    warm_trace, dropped = cowa.cowa_trace_entries()
    cowa.cowa_trace_start(0)
    cowa.cowa_get_device_error(dev)
    if dropped or not warm_trace:
        raise SystemExit("kernel trace of the warm-up incomplete")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    pairs = visible_pairs(wl.B, wl.Lq, wl.Lk, wl.Hq, wl.Hkv, quad, kv_head_offset=h0)
    dec_keys = decode_visible_keys([wl.Lk] * wl.B, wl.Hkv, quad, kv_head_offset=h0)
    work = kernel_work(wl, pairs, dec_keys)
    warm = {}
    for name, ms in warm_trace:
        n, tot = warm.get(name, (0, 0.0))
        warm[name] = (n + 1, tot + ms)
    top = max((n for n in warm if n in work), key=lambda n: warm[n][1])
    if world > 1:  # every rank times the same kernel
        top = sorted(work)[int(max_over_ranks([float(sorted(work).index(top))], world, dev)[0])]

    launches0 = cowa.cowa_launch_count()
    # the dominant kernel's launches in the timed steps get their own event pair
    cowa.cowa_trace_start(4 * args.steps + 16, only=top)
    with ClockSampler(local_rank) as clocks:
        for i in range(args.steps):
            flush.zero_()
            step(evs[i])
        torch.cuda.synchronize()
    cowa.cowa_trace_stop()
    launches = cowa.cowa_launch_count() - launches0
    trace, dropped = cowa.cowa_trace_entries()
    cowa.cowa_trace_start(0)
    if dropped or not trace:
        raise SystemExit("kernel trace of %s incomplete" % top)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    cowa.cowa_get_device_error(dev)

    t_fwd = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
    t_bwd = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
    t_dec = sum(e[2].elapsed_time(e[3]) for e in evs) / args.steps
    t_step = sum(e[0].elapsed_time(e[3]) for e in evs) / args.steps
    t_step, t_fwd, t_bwd, t_dec = max_over_ranks([t_step, t_fwd, t_bwd, t_dec], world, dev)

    g = wl.Hq // wl.Hkv
    # whole-job work: every rank's pairs and decode keys
    pairs_job, dec_keys_job = (int(x) for x in sum_over_ranks([pairs, dec_keys], world, dev))
    flops_job = pairs_job * 14 * wl.d + dec_keys_job * g * 4 * wl.d
    dec_bytes = dec_keys_job * 2 * wl.d * 2
    value = flops_job / (t_step * 1e-3) / 1e12

    # end to end through the public API from pinned host buffers
    e2e = run_e2e(args, cowa, wl, q, k, v, do, qd, seqlens, quad, h0, dev, stream, flush, world)
    e2e["value"] = flops_job / (e2e.pop("ms") * 1e-3) / 1e12
    e2e["unit"] = "TFLOP/s"

    # whole-job rates; the fractions are per GPU (job rate / N / peak)
    peaks, peak_src = load_peaks()
    long_step = t_step >= LONG_STEP_MS
    tensor_key = "bf16_tflops_sustained" if long_step else "bf16_tflops"
    tensor_peak = peaks[tensor_key]
    bwd_tflops = pairs_job * 10 * wl.d / (t_bwd * 1e-3) / 1e12
    fwd_tflops = pairs_job * 4 * wl.d / (t_fwd * 1e-3) / 1e12
    dec_gbs = dec_bytes / (t_dec * 1e-3) / 1e9

    # per-kernel shares from the traced warm-up steps; the roofline kernel's
    # time from its traced launches inside the timed steps
    names = sorted(warm)
    avg = max_over_ranks([warm[n][1] / warm[n][0] for n in names], world, dev)
    total = sum(warm[n][1] for n in names)
    kernels = {}
    for n, a in zip(names, avg):
        kernels[n] = {"launches": warm[n][0], "avg_ms": round(a, 5),
                      "share": round(warm[n][1] / total, 4)}
        if n in work:  # per GPU: rank 0's work over the slowest rank's time
            bound, amount, unit, _ = work[n]
            if bound == "tensor":
                kernels[n]["tflops"] = round(amount / (a * 1e-3) / 1e12, 2)
            else:
                kernels[n]["gbs"] = round(amount / (a * 1e-3) / 1e9, 1)
    bound, amount, unit, how = work[top]
    # per GPU: each rank's own work over its own average launch; the slowest
    # rank's rate is reported
    a_local = sum(ms for _, ms in trace) / len(trace)
    rate = amount / (a_local * 1e-3) / (1e12 if bound == "tensor" else 1e9)
    a_ms, neg_rate = max_over_ranks([a_local, -rate], world, dev)
    if bound == "tensor":
        achieved, peak, runit = -neg_rate, tensor_peak, "TFLOP/s"
        psrc = "%s %s (%s: the kernel runs %.2f ms inside a %.2f ms step, steps back to back)" % (
            peak_src, tensor_key, "sustained" if long_step else "burst", a_ms, t_step)
    else:
        achieved, peak, runit = -neg_rate, peaks["hbm_gbs"], "GB/s"
        psrc = "%s hbm_gbs" % peak_src
    roofline = {
        "kernel": top, "bound": bound, "achieved": round(achieved, 2), "peak": peak,
        "unit": runit, "frac": round(achieved / peak, 4), "peak_source": psrc,
        "frac_of_burst": round(achieved / peaks["bf16_tflops"], 4) if bound == "tensor" else None,
        "traffic": load_traffic(top, wl.name),
        "algorithmic": "%s per launch: %s" % (unit, how),
        "avg_launch_ms": round(a_ms, 5), "launches_timed": len(trace),
        "timing": "CUDA events around each launch of the kernel in the timed steps, on its stream",
    }
    result = {
        "metric": "effective TFLOP/s on visible pairs (fwd/bwd) & decode GB/s, % of B200 roofline",
        "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(t_step, 4), "higher_is_better": True,
        "scaling": "strong" if h0_mode(args, world) else "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic N(0,1), seeded",
        "config": {"workload": wl_job.name, "B": wl_job.B, "Lq": wl_job.Lq, "Lk": wl_job.Lk,
                   "Hq": wl_job.Hq, "Hkv": wl_job.Hkv, "d": wl_job.d, "quad": list(quad),
                   "step": "cowa_fwd + cowa_bwd + cowa_decode(last token, full K/V as cache)",
                   "l2": "512 MiB write before every timed step",
                   "parallelism": ("kv-heads%d (rank r: KV heads [r*%d, (r+1)*%d), kv_head_offset = r*%d)"
                                   % (world, wl.Hkv, wl.Hkv, wl.Hkv)) if h0_mode(args, world)
                   else "dp%d (independent replicas)" % world},
        "breakdown": {
            "fwd_ms": round(t_fwd, 4), "fwd_tflops": round(fwd_tflops, 2),
            "fwd_frac": round(fwd_tflops / world / tensor_peak, 4),
            "bwd_ms": round(t_bwd, 4), "bwd_tflops": round(bwd_tflops, 2),
            "bwd_frac": round(bwd_tflops / world / tensor_peak, 4),
            "tensor_peak": tensor_peak, "tensor_peak_source": "%s %s" % (peak_src, tensor_key),
            "fwd_frac_of_burst": round(fwd_tflops / world / peaks["bf16_tflops"], 4),
            "bwd_frac_of_burst": round(bwd_tflops / world / peaks["bf16_tflops"], 4),
            "decode_ms": round(t_dec, 4), "decode_gbs": round(dec_gbs, 1),
            "decode_frac": round(dec_gbs / world / peaks["hbm_gbs"], 4),
            "visible_pairs": pairs_job, "decode_visible_keys": dec_keys_job,
            "kernels": kernels,
            "kernels_from": "CUDA events around every library launch of the traced warm-up steps",
        },
        "roofline": roofline,
        "clocks": clocks.summary(),
        "e2e": e2e,
        "gpu_launches": int(launches),
    }
    if args.packed:
        result["packed_workload"] = run_packed_workload(args, cowa, wl, h0, dev, stream, flush, world, peaks)
    if args.full_mask:
        result["full_mask_control"] = run_full_mask(args, cowa, wl, q, k, v, do, qd, seqlens, h0, dev, stream,
                                                    flush, world, (t_fwd, t_bwd, t_dec))
    if args.decode_workload:
        result["decode_workload"] = run_decode_workload(args, cowa, rank, dev, stream, flush, world, peaks,
                                                        peak_src)
    if args.mala and not h0_mode(args, world):
        result["mala_workload"] = run_mala_workload(args, cowa, rank, dev, stream, flush, world, peaks,
                                                    tensor_peak)
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        result["cpu_baseline"] = run_cpu_baseline(wl, q, k, v, do, quad, args.cpu_rows)
    return result


def run_e2e(args, cowa, wl, q, k, v, do, qd, seqlens, quad, h0, dev, stream, flush, world):
    """The step through the public API with its inputs copied in from pinned
    host memory and all of its results copied back, every step.  Steps are
    pipelined as an application would run them: two sets of device buffers
    (step i uses set i % 2) and three streams, so step i+1's inputs arrive
    and step i-1's results leave while step i computes; events keep each set
    from being overwritten while a copy or a kernel still reads it.  The L2
    flush precedes every step's kernels.  Time per step = (end of the last
    copy back - start of the first copy in) / steps."""
    import torch.distributed as dist
    srcs = [t.cpu().pin_memory() for t in (q, k, v, do, qd, seqlens)]
    outs = {"o": torch.empty(q.shape, dtype=q.dtype).pin_memory(),
            "dq": torch.empty(q.shape, dtype=q.dtype).pin_memory(),
            "dk": torch.empty(k.shape, dtype=k.dtype).pin_memory(),
            "dv": torch.empty(v.shape, dtype=v.dtype).pin_memory(),
            "od": torch.empty(qd.shape, dtype=qd.dtype).pin_memory()}
    h2d = sum(t.numel() * t.element_size() for t in srcs)
    d2h = sum(t.numel() * t.element_size() for t in outs.values())
    B, Lq, Hq = q.shape[0], q.shape[1], q.shape[2]
    sets = []
    for _ in range(2):
        ins = [torch.empty(t.shape, dtype=t.dtype, device=dev) for t in srcs]
        sets.append({"ins": ins, "o": torch.empty_like(ins[0]),
                     "lse": torch.empty((B, Hq, Lq), dtype=torch.float32, device=dev),
                     "dq": torch.empty_like(ins[0]), "dk": torch.empty_like(ins[1]), "dv": torch.empty_like(ins[2]),
                     "od": torch.empty_like(ins[4]), "lsed": torch.empty((B, Hq), dtype=torch.float32, device=dev),
                     "free_in": None, "free_out": None})
    ws_f = torch.empty(cowa.cowa_fwd_workspace_size(q, k, quad, h0), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(cowa.cowa_bwd_workspace_size(q, k, quad, h0), dtype=torch.uint8, device=dev)
    ws_d = torch.empty(cowa.cowa_decode_workspace_size(qd, k, quad, h0), dtype=torch.uint8, device=dev)
    s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))

    def e2e_step(i):
        st = sets[i % 2]
        with torch.cuda.stream(s_in):
            if st["free_in"] is not None:  # step i-2's kernels have read this set's inputs
                s_in.wait_event(st["free_in"])
            for dst, src in zip(st["ins"], srcs):
                dst.copy_(src, non_blocking=True)
            landed = torch.cuda.Event()
            landed.record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(landed)
            if st["free_out"] is not None:  # step i-2's results have left this set
                s_cmp.wait_event(st["free_out"])
            flush.zero_()
            q_, k_, v_, do_, qd_, sl_ = st["ins"]
            cowa.cowa_fwd(q_, k_, v_, quad, kv_head_offset=h0, out=st["o"], lse=st["lse"], workspace=ws_f)
            cowa.cowa_bwd(q_, k_, v_, st["o"], st["lse"], do_, quad, kv_head_offset=h0,
                          dq=st["dq"], dk=st["dk"], dv=st["dv"], workspace=ws_b)
            cowa.cowa_decode(qd_, k_, v_, sl_, quad, kv_head_offset=h0, out=st["od"], lse=st["lsed"],
                             workspace=ws_d)
            done = torch.cuda.Event()
            done.record(s_cmp)
            st["free_in"] = done
        with torch.cuda.stream(s_out):
            s_out.wait_event(done)
            for name in ("o", "dq", "dk", "dv", "od"):
                outs[name].copy_(st[name], non_blocking=True)
            back = torch.cuda.Event()
            back.record(s_out)
            st["free_out"] = back

    for i in range(max(1, args.warmup)):
        e2e_step(i)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0.record(s_in)
    for i in range(args.steps):
        e2e_step(i)
    t1.record(s_out)
    torch.cuda.synchronize()
    ms = max_over_ranks([t0.elapsed_time(t1) / args.steps], world, dev)[0]
    return {"ms": ms, "ms_per_step": round(ms, 4),
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "path": "pinned host -> device copies, cowa_fwd/bwd/decode, device -> pinned host, every step; "
                    "neighbouring steps' copies overlap the compute (two device buffer sets, three streams)"}


def run_full_mask(args, cowa, wl, q, k, v, do, qd, seqlens, h0, dev, stream, flush, world, t_cowa):
    """The same step with the full-causal quadruple (0, Lk, 0, 0): every key
    at distance 0 .. p is visible to every head.  The ratio of the two times
    is the speedup over a full causal mask, bounded by the ratio of visible
    work (full-causal pairs / CoWA pairs)."""
    import torch.distributed as dist
    quad = (0, wl.Lk, 0, 0)
    o = torch.empty_like(q)
    lse = torch.empty((wl.B, wl.Hq, wl.Lq), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    od = torch.empty_like(qd)
    lsed = torch.empty((wl.B, wl.Hq), dtype=torch.float32, device=dev)
    ws_f = torch.empty(cowa.cowa_fwd_workspace_size(q, k, quad), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(cowa.cowa_bwd_workspace_size(q, k, quad), dtype=torch.uint8, device=dev)
    ws_d = torch.empty(cowa.cowa_decode_workspace_size(qd, k, quad), dtype=torch.uint8, device=dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        cowa.cowa_fwd(q, k, v, quad, out=o, lse=lse, workspace=ws_f)
        if ev is not None:
            ev[1].record(stream)
        cowa.cowa_bwd(q, k, v, o, lse, do, quad, dq=dq, dk=dk, dv=dv, workspace=ws_b)
        if ev is not None:
            ev[2].record(stream)
        cowa.cowa_decode(qd, k, v, seqlens, quad, out=od, lse=lsed, workspace=ws_d)
        if ev is not None:
            ev[3].record(stream)

    steps = max(3, min(args.steps, 10))
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    if world > 1:
        dist.barrier()
    for i in range(steps):
        flush.zero_()
        step(evs[i])
    torch.cuda.synchronize()
    cowa.cowa_get_device_error(dev)
    t = [sum(e[a].elapsed_time(e[a + 1]) for e in evs) / steps for a in range(3)]
    t = max_over_ranks(t, world, dev)
    # whole-job work ratios; with KV-head sharding the slowest rank (the
    # lowest heads, whose long windows lie nearest and are seen by the most
    # query rows) bounds the speedup instead
    full_pairs, cowa_pairs, full_keys, cowa_keys = sum_over_ranks([
        visible_pairs(wl.B, wl.Lq, wl.Lk, wl.Hq, wl.Hkv, quad),
        visible_pairs(wl.B, wl.Lq, wl.Lk, wl.Hq, wl.Hkv, wl.quad, kv_head_offset=h0),
        decode_visible_keys([wl.Lk] * wl.B, wl.Hkv, quad),
        decode_visible_keys([wl.Lk] * wl.B, wl.Hkv, wl.quad, kv_head_offset=h0)], world, dev)
    return {"quad": list(quad), "steps": steps,
            "fwd_ms": round(t[0], 4), "bwd_ms": round(t[1], 4), "decode_ms": round(t[2], 4),
            "speedup_fwd": round(t[0] / t_cowa[0], 3), "speedup_bwd": round(t[1] / t_cowa[1], 3),
            "speedup_decode": round(t[2] / t_cowa[2], 3),
            "visible_work_ratio_fwd_bwd": round(full_pairs / cowa_pairs, 3),
            "visible_work_ratio_decode": round(full_keys / cowa_keys, 3)}


def packed_lengths(total, lo, hi, seed):
    """Seeded ragged sequence lengths, log-uniform in [lo, hi], summing to total."""
    rng = np.random.default_rng(seed)
    out = []
    while sum(out) < total:
        n = int(round(float(np.exp(rng.uniform(np.log(lo), np.log(hi))))))
        out.append(min(n, total - sum(out)))
    return out


def run_packed_workload(args, cowa, wl, h0, dev, stream, flush, world, peaks):
    """A packed (variable-length) batch with the workload's heads and window
    quadruple: as many tokens as the workload's batch, in sequences of
    log-uniform lengths between 1/16 and 1x the workload's length."""
    import torch.distributed as dist
    from structured_sparse_attention_block_b200.inputs import training_inputs
    lens = packed_lengths(wl.B * wl.Lq, max(1, wl.Lq // 16), wl.Lq, seed=17)
    T = sum(lens)
    q, k, v, do = (t[0] for t in training_inputs(1, T, T, wl.Hq, wl.Hkv, wl.d, device=dev, seed=23))
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32), device=dev)
    mx = max(lens)
    pairs = int(sum_over_ranks([sum(visible_pairs(1, n, n, wl.Hq, wl.Hkv, wl.quad, kv_head_offset=h0)
                                    for n in lens)], world, dev)[0])
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(max(3, args.steps))]

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        o, lse = cowa.cowa_fwd_varlen(q, k, v, cu, cu, mx, mx, wl.quad, kv_head_offset=h0)
        if ev is not None:
            ev[1].record(stream)
        cowa.cowa_bwd_varlen(q, k, v, o, lse, do, cu, cu, mx, mx, wl.quad, kv_head_offset=h0)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    for ev in evs:
        flush.zero_()
        step(ev)
    torch.cuda.synchronize()
    cowa.cowa_get_device_error(dev)
    t_f, t_b = max_over_ranks([sum(e[0].elapsed_time(e[1]) for e in evs) / len(evs),
                               sum(e[1].elapsed_time(e[2]) for e in evs) / len(evs)], world, dev)
    fwd_tf = pairs * 4 * wl.d / (t_f * 1e-3) / 1e12
    bwd_tf = pairs * 10 * wl.d / (t_b * 1e-3) / 1e12
    return {"sequences": len(lens), "tokens": T, "min_len": min(lens), "max_len": mx,
            "visible_pairs": pairs, "fwd_ms": round(t_f, 4), "bwd_ms": round(t_b, 4),
            "fwd_tflops": round(fwd_tf, 2), "bwd_tflops": round(bwd_tf, 2),
            "fwd_frac": round(fwd_tf / world / peaks["bf16_tflops"], 4),
            "bwd_frac": round(bwd_tf / world / peaks["bf16_tflops"], 4),
            "lengths": "log-uniform in [L/16, L], seed 17"}


def run_decode_workload(args, cowa, rank, dev, stream, flush, world, peaks, peak_src):
    """The 128K decode workload (B=16, Hq=32, Hkv=8, d=128), timed on its own
    (whole-job bytes over the slowest rank's time; fractions per GPU)."""
    import torch.distributed as dist
    from structured_sparse_attention_block_b200.inputs import WORKLOADS, workload_inputs
    wl, h0 = head_shard(WORKLOADS["decode128k"], rank, world, args.parallel)
    q, kc, vc, sl = workload_inputs(wl, device=dev, seed=7 + 1000 * rank)
    out = torch.empty_like(q)
    lse = torch.empty((wl.B, wl.Hq), dtype=torch.float32, device=dev)
    ws = torch.empty(cowa.cowa_decode_workspace_size(q, kc, wl.quad, h0), dtype=torch.uint8, device=dev)
    for _ in range(max(3, args.warmup)):
        cowa.cowa_decode(q, kc, vc, sl, wl.quad, kv_head_offset=h0, out=out, lse=lse, workspace=ws)
    torch.cuda.synchronize()
    n = max(args.steps, 10)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    if world > 1:
        dist.barrier()
    for i in range(n):
        flush.zero_()
        evs[i][0].record(stream)
        cowa.cowa_decode(q, kc, vc, sl, wl.quad, kv_head_offset=h0, out=out, lse=lse, workspace=ws)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks([sum(a.elapsed_time(b) for a, b in evs) / n], world, dev)[0]
    keys = int(sum_over_ranks([decode_visible_keys([wl.Lk] * wl.B, wl.Hkv, wl.quad, kv_head_offset=h0)],
                              world, dev)[0])
    nbytes = keys * 2 * wl.d * 2
    gbs = nbytes / (ms * 1e-3) / 1e9

    # the same decode over a windowed cache built for the next `horizon` steps:
    # each KV head holds only the keys those steps see
    horizon = 64
    origin = sl - 1
    kw, vw = cowa.cowa_wcache_build(kc, vc, origin, wl.quad, horizon, kv_head_offset=h0)
    del kc, vc
    torch.cuda.empty_cache()
    for _ in range(max(3, args.warmup)):
        cowa.cowa_decode_windowed(q, kw, vw, sl, origin, wl.quad, horizon, kv_head_offset=h0,
                                  out=out, lse=lse, workspace=ws)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    for i in range(n):
        flush.zero_()
        evs[i][0].record(stream)
        cowa.cowa_decode_windowed(q, kw, vw, sl, origin, wl.quad, horizon, kv_head_offset=h0,
                                  out=out, lse=lse, workspace=ws)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    cowa.cowa_get_device_error(dev)
    ms_w = max_over_ranks([sum(a.elapsed_time(b) for a, b in evs) / n], world, dev)[0]
    full_bytes, win_bytes = (int(x) for x in sum_over_ranks(
        [wl.B * wl.Lk * wl.Hkv * wl.d * 2 * 2, kw.numel() * kw.element_size() * 2], world, dev))
    del q, kw, vw
    torch.cuda.empty_cache()
    return {"workload": wl.name, "ms": round(ms, 4), "visible_kv_bytes": nbytes,
            "GB/s": round(gbs, 1), "peak": peaks["hbm_gbs"], "frac": round(gbs / world / peaks["hbm_gbs"], 4),
            "peak_source": "%s hbm_gbs" % peak_src,
            "full_cache_bytes": full_bytes,
            "windowed": {"horizon": horizon, "cache_bytes": win_bytes,
                         "memory_ratio": round(full_bytes / win_bytes, 3), "ms": round(ms_w, 4),
                         "GB/s": round(nbytes / (ms_w * 1e-3) / 1e9, 1)}}


def mala_pair_counts(keep, Lq, Lk, bm=128, bn=64):
    """(causal pairs, kept pairs) over all (b, hq) of a MALA decision array
    keep [B, Hq, nqt, nkt]: a block's pairs are (i, j) with j <= i + Lk - Lq."""
    nqt, nkt = keep.shape[2], keep.shape[3]
    p = np.arange(Lq, dtype=np.int64) + (Lk - Lq)
    per_block = np.zeros((nqt, nkt), dtype=np.int64)
    for t in range(nkt):
        j0, j1 = t * bn, min((t + 1) * bn, Lk)
        cnt = np.clip(np.minimum(p + 1, j1) - j0, 0, None)  # keys of block t row i sees
        per_block[:, t] = np.add.reduceat(cnt, np.arange(0, Lq, bm))
    causal = int(per_block.sum()) * keep.shape[0] * keep.shape[1]
    kept = int((keep.astype(np.int64) * per_block[None, None]).sum())
    return causal, kept


def run_mala_workload(args, cowa, rank, dev, stream, flush, world, peaks, tensor_peak):
    """MALA (the pages' companion operator: full causal scoring, blocks of
    128 query rows x 64 keys kept when some row gives them at least tau of
    its softmax mass) on the 14B-like 32K shape, where the pages quote its
    training-FLOP saving; forward and backward timed separately.  Work is
    counted per the reading: forward 2d per causal pair (scoring) + 2d per
    kept pair (PV); backward 6d per causal pair (S, dQ, dK) + 4d per kept
    pair (dP, dV)."""
    import torch.distributed as dist
    from structured_sparse_attention_block_b200.inputs import WORKLOADS, workload_inputs
    wl = WORKLOADS["llm14b_32k"]
    tau = 2.0 ** -8
    q, k, v, do = workload_inputs(wl, seed=11 + 1000 * rank)
    o, lse, keep = cowa.cowa_mala_fwd(q, k, v, tau)
    ws = torch.empty(cowa.lib().cowa_mala_bwd_workspace_size(
        ctypes_shape(cowa, q, k, v, o)), dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        cowa.cowa_mala_fwd(q, k, v, tau, out=o, lse=lse, keep=keep)
        cowa.cowa_mala_bwd(q, k, v, o, lse, keep, do, workspace=ws)
    torch.cuda.synchronize()
    n = max(3, min(args.steps, 10))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n)]
    if world > 1:
        dist.barrier()
    for e in evs:
        flush.zero_()
        e[0].record(stream)
        cowa.cowa_mala_fwd(q, k, v, tau, out=o, lse=lse, keep=keep)
        e[1].record(stream)
        cowa.cowa_mala_bwd(q, k, v, o, lse, keep, do, workspace=ws)
        e[2].record(stream)
    torch.cuda.synchronize()
    cowa.cowa_get_device_error(dev)
    t_f, t_b = max_over_ranks([sum(e[0].elapsed_time(e[1]) for e in evs) / n,
                               sum(e[1].elapsed_time(e[2]) for e in evs) / n], world, dev)
    causal, kept = mala_pair_counts(keep.cpu().numpy(), wl.Lq, wl.Lk)
    causal, kept = (int(x) for x in sum_over_ranks([causal, kept], world, dev))
    fwd_fl = causal * 2 * wl.d + kept * 2 * wl.d
    bwd_fl = causal * 6 * wl.d + kept * 4 * wl.d
    del q, k, v, do, o, lse, keep, ws
    torch.cuda.empty_cache()
    return {"workload": wl.name, "tau": tau, "block": [128, 64],
            "causal_pairs": causal, "kept_pairs": kept, "kept_fraction": round(kept / causal, 4),
            "fwd_ms": round(t_f, 4), "bwd_ms": round(t_b, 4),
            "fwd_tflops": round(fwd_fl / (t_f * 1e-3) / 1e12, 2), "bwd_tflops": round(bwd_fl / (t_b * 1e-3) / 1e12, 2),
            "fwd_frac": round(fwd_fl / (t_f * 1e-3) / 1e12 / world / tensor_peak, 4),
            "bwd_frac": round(bwd_fl / (t_b * 1e-3) / 1e12 / world / tensor_peak, 4),
            "counted": "fwd 2d/causal pair + 2d/kept pair; bwd 6d/causal pair + 4d/kept pair",
            "inputs": "synthetic N(0,1): attention is diffuse, so a block's mass falls with the row's length"}


def ctypes_shape(cowa, q, k, v, o):
    import ctypes
    return ctypes.byref(cowa._shape(q, k, v, o, 0))


# ------------------------------------------------------------ CPU oracle ----
def oracle_sample(wl, q, k, v, do, quad, rows):
    """The oracle on a bounded sample of the step: batch element 0, the last
    `rows` query rows (a chunk of the same problem under bottom-right
    alignment), forward + backward, plus one decode row per query head.
    Returns (seconds, flops credited to the sample, threads)."""
    from oracle import oracle
    from structured_sparse_attention_block_b200.inputs import bf16_bits
    Lq = wl.Lq
    rows = min(rows, Lq)
    qb = bf16_bits(q[:1, Lq - rows:])
    kb, vb = bf16_bits(k[:1]), bf16_bits(v[:1])
    db = bf16_bits(do[:1, Lq - rows:])
    t0 = time.perf_counter()
    oracle.fwd(qb, kb, vb, quad)
    oracle.bwd(qb, kb, vb, db, quad)
    oracle.decode(bf16_bits(q[:1, -1]), kb, vb, [wl.Lk], quad)
    sec = time.perf_counter() - t0
    pairs = visible_pairs(1, wl.Lq, wl.Lk, wl.Hq, wl.Hkv, quad, rows=np.arange(Lq - rows, Lq))
    dec = decode_visible_keys([wl.Lk], wl.Hkv, quad) * (wl.Hq // wl.Hkv)
    flops = pairs * 14 * wl.d + dec * 4 * wl.d
    return sec, flops, oracle.threads(), rows


def run_cpu_baseline(wl, q, k, v, do, quad, rows):
    sec, flops, thr, rows = oracle_sample(wl, q, k, v, do, quad, rows)
    return {"value": flops / sec / 1e12, "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
            "seconds": round(sec, 2),
            "sample": "batch 0, last %d of %d query rows, all heads: fp64 forward + backward "
                      "+ one decode row per head" % (rows, wl.Lq)}


def run_reference(args, rank, world):
    """The reference arm: the fp64 oracle as it stands, on host cores."""
    if rank != 0:
        return None
    from structured_sparse_attention_block_b200.inputs import WORKLOADS, training_inputs
    wl = WORKLOADS[args.workload]
    q, k, v, do = training_inputs(1, wl.Lq, wl.Lk, wl.Hq, wl.Hkv, wl.d, device="cpu", seed=0)
    rows = args.ref_rows
    for _ in range(args.warmup):
        oracle_sample(wl, q, k, v, do, wl.quad, rows)
    secs, flops, thr = 0.0, 0, 1
    for _ in range(args.steps):
        s, f, thr, rows = oracle_sample(wl, q, k, v, do, wl.quad, rows)
        secs += s
        flops += f
    value = flops / secs / 1e12
    ms = secs / args.steps * 1e3
    sample = ("batch 0, last %d of %d query rows, all heads: fp64 forward + backward + one "
              "decode row per head" % (rows, wl.Lq))
    return {
        "impl": "reference",
        "metric": "effective TFLOP/s on visible pairs (fwd/bwd) & decode GB/s, % of B200 roofline",
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 2), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic N(0,1), seeded",
        "config": {"workload": wl.name, "B": wl.B, "Lq": wl.Lq, "Lk": wl.Lk, "Hq": wl.Hq, "Hkv": wl.Hkv,
                   "d": wl.d, "quad": list(wl.quad), "parallelism": "host cores (OpenMP)"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": thr, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["cowa", "reference"], default="cowa")
    ap.add_argument("--workload", default="op128k")
    ap.add_argument("--parallel", choices=["dp", "heads"], default="dp",
                    help="dp: one replica per GPU (weak scaling); heads: KV heads sharded over the GPUs "
                         "with kv_head_offset (strong scaling)")
    ap.add_argument("--cpu-rows", type=int, default=None,
                    help="query rows in the CPU-baseline sample (default: per workload, about 10-20 s of "
                         "oracle work on 16 cores)")
    ap.add_argument("--ref-rows", type=int, default=None,
                    help="query rows per reference-arm step (default: per workload, a few seconds each)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode-workload", dest="decode_workload", action="store_false")
    ap.add_argument("--no-packed", dest="packed", action="store_false",
                    help="skip the packed variable-length batch of the workload's heads and windows")
    ap.add_argument("--no-full-mask", dest="full_mask", action="store_false",
                    help="skip the full-causal-mask control run of the same step")
    ap.add_argument("--no-mala", dest="mala", action="store_false",
                    help="skip the MALA forward + backward leg (14B-like 32K shape)")
    args = ap.parse_args()
    if args.cpu_rows is None:
        args.cpu_rows = CPU_ROWS.get(args.workload, 256)
    if args.ref_rows is None:
        args.ref_rows = REF_ROWS.get(args.workload, 64)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            raise SystemExit("--gpus %d needs torchrun with %d processes" % (args.gpus, args.gpus))
        raise SystemExit("WORLD_SIZE=%d does not match --gpus %d" % (world, args.gpus))

    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    import torch.distributed as dist
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        res = run_cowa(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
