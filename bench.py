#!/usr/bin/env python3
"""Benchmark of the quantized-KV decode step (K4V2) on B200.

A step is one pass of the hot path over one batch: append one new token per
sequence through kvq_quantize_append (the token leaving the bf16 window is
quantized into its page, the new one enters the window) and then
kvq_decode_attention of one query token per sequence over the whole cache
(fused dequantization, GQA, online softmax, split-K combine).

Default workload: Llama-3-8B-shaped layer, batch 16, 32 query / 8 KV heads,
head_dim 128, 4096 cached tokens after the append, K4 g32 / V2 g128, 128
newest tokens in bf16.  Inputs are seeded synthetic data.  Several copies of
the cache are rotated so that the bytes touched between two reads of the
same copy exceed twice the L2 size; each step reads HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference     # the CPU oracle on the host cores

Prints one JSON line (rank 0).  With N > 1 (torchrun) every rank runs an
independent replica on its own GPU (the path has no exchange step); the
step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "quantized-KV decode attention µs/step and HBM GB/s (% of B200 peak), K4V2"
WORKLOADS = {"llama8b": wl.LLAMA8B, "ragged": wl.RAGGED,
             "rotation": wl.ROTATION, "tiny": wl.TINY,
             # the memory-budget planner's pick at 116 B per token-head: key groups of 64 positions
             "per_channel_llama8b": wl.LLAMA8B.with_(name="llama3_8b_layer_b16_l4096_k4pc64v2g64_w128",
                                                     k_group=64, v_group=64, k_per_channel=True),
             # eight query heads per kv-head (the decode kernel's eight-head build), 64 of them
             "per_channel_gqa8": wl.LLAMA8B.with_(name="b16_l4096_q64kv8_k4pc64v2g64_w128", num_q_heads=64,
                                                  k_group=64, v_group=64, k_per_channel=True),
             # the same layout at long context, few pairs (8 x 8): each pair split between CTAs
             "per_channel_sweep": wl.SWEEP.with_(name="sweep_b8_l16384_k4pc64v2g64_w0", k_bits=4, v_bits=2,
                                                 k_group=64, v_group=64, k_per_channel=True)}
# the long-context bit-allocation sweep: one workload per (key bits, value bits)
WORKLOADS.update({f"sweep_k{v.k_bits}v{v.v_bits}": v for v in wl.sweep_variants()})
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_HBM_GBS = 6650.0
# chunked-prefill attention: (cache shape, queries per sequence in the chunk)
PREFILL_WORKLOADS = {"prefill_llama8b": (wl.LLAMA8B, 512)}
PREFILL_METRIC = "chunked-prefill attention over the quantized cache, µs/step (fp32 TFLOP/s)"


# ------------------------------------------------------------------ shared

def paged_positions(w: wl.Workload, L: int) -> int:
    """Positions of a length-L sequence that live in pages: below L - W, and
    whole key groups only when key groups run along positions."""
    q = max(0, L - w.window)
    return q - q % w.k_group if w.k_per_channel else q


def algorithmic_bytes(w: wl.Workload, lens) -> int:
    """Bytes the decode attention must read: packed codes + fp16 metadata of
    every quantized token and bf16 K/V of every window token, per kv-head.
    (Key metadata per token and kv-head is 4*d/k_group bytes for groups of
    k_group channels and for groups of k_group positions alike.)"""
    d = w.head_dim
    t = d * w.k_bits // 8 + 4 * d // w.k_group + d * w.v_bits // 8 + 4 * d // w.v_group
    total = 0
    for L in lens:
        L = int(L)
        q = paged_positions(w, L)
        total += (q * t + (L - q) * 4 * d) * w.num_kv_heads
    return total


def measured_hbm_peak():
    for p in (os.path.join(ROOT, "MEASURED_PEAKS.json"),):
        try:
            with open(p) as f:
                v = json.load(f).get("hbm_gbs")
            if v:
                return float(v), "measured"
        except (OSError, ValueError):
            pass
    return FALLBACK_HBM_GBS, "fallback"


def measured_bf16_peak():
    """Dense bf16 tensor peak (TFLOP/s) for a kernel timed alone: the measured
    burst figure of MEASURED_PEAKS.json, else the fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            v = json.load(f).get("bf16_tflops")
        if v:
            return float(v), "measured"
    except (OSError, ValueError):
        pass
    return FALLBACK_BF16_TFLOPS, "fallback"


def prefill_on_tensor_cores(w) -> bool:
    """The layouts the library's tensor-core prefill kernel takes (head_dim 128,
    key groups of 32 channels of a token, unrotated keys, value groups dividing
    128); the others run on CUDA cores."""
    return (w.head_dim == 128 and not w.k_per_channel and not w.rotate_keys and w.k_group == 32
            and 128 % w.v_group == 0)


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_dist(backend: str):
    ws, rank, local = dist_env()
    if ws <= 1:
        return None
    import datetime
    import torch.distributed as dist
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def reduce_max(dist, value: float, device=None) -> float:
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def cache_lens(w: wl.Workload):
    """Tokens attended per step; the cache holds one fewer before the append."""
    final = wl.lengths(w).astype(np.int32)
    return final - 1, final


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi clock / throttle samples taken while the GPU works."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, interval_ms: int = 50):
        self.gpu = gpu_index
        self.interval = interval_ms
        self.proc = None
        self.lines = []
        self.mark = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 f"-lms", str(self.interval), "-i", str(self.gpu)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)

    def summary(self, t0: float, t1: float):
        if self.proc is None:
            return None
        rows = []
        for ts, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((ts, float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        window = [r for r in rows if t0 <= r[0] <= t1]
        used = window if window else rows
        if not used:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in used for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": float(np.median([r[1] for r in used])), "sm_max_mhz": max(r[2] for r in used),
                "reasons": reasons, "samples": len(used),
                "window": "timed region" if window else "whole run (timed region shorter than one sample)"}


# ------------------------------------------------------------------ oracle (CPU)

def oracle_step_timer(w: wl.Workload, budget_s: float):
    """Time the CPU oracle (as it stands) on full steps of the workload for
    about `budget_s` seconds of work: append one token per sequence, then
    fp64 decode attention for every query head.  Returns (us_per_step, cores,
    sample description)."""
    import oracle
    lens0, lens1 = cache_lens(w)
    kr, vr, _, _, cu, _ = wl.prefill(w, lens0, with_f32=False)
    pt = wl.page_table(w, np.maximum(0, lens1 - w.window))
    signs = wl.rotation_signs(w) if w.rotate_keys else None
    c = oracle.Cache(oracle.Layout.from_workload(w, signs), w.batch, pt, max(1, int((pt >= 0).sum())))
    in_dt = oracle.IN_BF16 if w.in_dtype == wl.DT_BF16 else oracle.IN_F32
    c.append(kr, vr, in_dt, cu, np.zeros(w.batch, np.int32))
    del kr, vr
    cu1 = np.arange(w.batch + 1, dtype=np.int32)
    times = []
    first = None
    t_all = time.perf_counter()
    i = 0
    while True:
        k1, v1, _, _ = wl.new_tokens(w, i)
        qr, _ = wl.query(w, i)
        t = time.perf_counter()
        c.append(k1, v1, in_dt, cu1, lens0)
        o, _ = c.decode_attention(qr, in_dt, lens1, 1.0 / math.sqrt(w.head_dim))
        times.append(time.perf_counter() - t)
        if first is None:
            first = np.array(o, np.float64)
        i += 1
        if (time.perf_counter() - t_all >= budget_s and i >= 2) or i >= 1000:
            break
    us = float(np.mean(times)) * 1e6
    return us, oracle.num_threads(), f"{i} full steps of {w.name} (append + fp64 attention, all heads)", first


def oracle_tiny_single_thread(steps: int = 20):
    """The oracle on one thread, on the tiny configuration (1 sequence of 256
    tokens, 4/4 heads, d64, K4V2, fp32 inputs): mean microseconds of a full
    step (append one token, fp64 attention of every head)."""
    import oracle
    before = oracle.num_threads()
    oracle.set_num_threads(1)
    try:
        us, _, _ = _tiny_steps(steps)
    finally:
        oracle.set_num_threads(before)
    return us


def _tiny_steps(steps: int):
    import oracle
    w = wl.TINY
    lens0, lens1 = cache_lens(w)
    kr, vr, _, _, cu, _ = wl.prefill(w, lens0, with_f32=False)
    pt = wl.page_table(w, np.maximum(0, lens1 - w.window))
    c = oracle.Cache(oracle.Layout.from_workload(w), w.batch, pt, max(1, int((pt >= 0).sum())))
    in_dt = oracle.IN_BF16 if w.in_dtype == wl.DT_BF16 else oracle.IN_F32
    c.append(kr, vr, in_dt, cu, np.zeros(w.batch, np.int32))
    cu1 = np.arange(w.batch + 1, dtype=np.int32)
    times = []
    for i in range(steps):
        k1, v1, _, _ = wl.new_tokens(w, i)
        qr, _ = wl.query(w, i)
        t = time.perf_counter()
        c.append(k1, v1, in_dt, cu1, lens0)
        c.decode_attention(qr, in_dt, lens1, 1.0 / math.sqrt(w.head_dim))
        times.append(time.perf_counter() - t)
    return float(np.median(times)) * 1e6, 1, ""


def run_reference(args):
    ws, rank, local = dist_env()
    dist = init_dist("gloo")
    w = WORKLOADS[args.workload]
    if rank != 0:
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()
        return
    import oracle
    lens0, lens1 = cache_lens(w)
    kr, vr, _, _, cu, _ = wl.prefill(w, lens0, with_f32=False)
    pt = wl.page_table(w, np.maximum(0, lens1 - w.window))
    signs = wl.rotation_signs(w) if w.rotate_keys else None
    c = oracle.Cache(oracle.Layout.from_workload(w, signs), w.batch, pt, max(1, int((pt >= 0).sum())))
    in_dt = oracle.IN_BF16 if w.in_dtype == wl.DT_BF16 else oracle.IN_F32
    c.append(kr, vr, in_dt, cu, np.zeros(w.batch, np.int32))
    del kr, vr
    # a bounded sample per step: every query head of `sample_b` sequences
    sample_b = max(1, min(w.batch, int(args.ref_sample_seqs)))
    cu1 = np.arange(w.batch + 1, dtype=np.int32)
    sub_lens = lens1.copy()
    sub_lens[sample_b:] = 0            # only the sampled sequences attend

    def step(i):
        k1, v1, _, _ = wl.new_tokens(w, i)
        qr, _ = wl.query(w, i)
        t = time.perf_counter()
        c.append(k1, v1, in_dt, cu1, lens0)
        c.decode_attention(qr, in_dt, sub_lens, 1.0 / math.sqrt(w.head_dim))
        return time.perf_counter() - t

    for i in range(args.warmup):
        step(i)
    total = 0.0
    for i in range(args.steps):
        total += step(args.warmup + i)
    scale = w.batch / sample_b
    us = total / max(1, args.steps) * 1e6 * scale
    sample = (f"each step: append 1 token x {w.batch} seqs + fp64 attention of all query heads of "
              f"{sample_b}/{w.batch} sequences, time scaled by {scale:g}")
    line = {"impl": "reference", "metric": METRIC, "value": us, "unit": "us/step", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": us / 1e3,
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w, lens1),
            "cpu_baseline": {"value": us, "unit": "us/step", "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": sample,
                             "tiny_single_thread_us": oracle_tiny_single_thread()},
            "e2e": {"value": us, "unit": "us/step", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def workload_config(w: wl.Workload, lens1) -> dict:
    cfg = {"workload": w.name, "batch": w.batch, "q_heads": w.num_q_heads, "kv_heads": w.num_kv_heads,
           "head_dim": w.head_dim, "k_bits": w.k_bits, "v_bits": w.v_bits, "k_group": w.k_group,
           "v_group": w.v_group, "window": w.window, "page_size": w.page_size,
           "rotate_keys": bool(w.rotate_keys), "k_per_channel": bool(w.k_per_channel),
           "tokens_attended": int(lens1[0]) if w.ragged is None else "ragged",
           "total_tokens": int(np.sum(lens1)),
           "step": "append 1 token per sequence + decode attention (1 query token per sequence), one kvq_append_decode call",
           "parallelism": "replicas (no exchange step)"}
    return cfg


# ------------------------------------------------------------------ ours (GPU)

def source_digest(paths) -> str:
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profile_traffic(workload: str):
    """Per-launch DRAM traffic of the decode kernels from the committed ncu
    summary, if it was taken on the current kernel sources."""
    path = os.path.join(ROOT, "profiles", f"decode_attention_{workload}.txt")
    try:
        kv = {}
        for line in open(path):
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
        srcs = kv.get("sources", "").split()
        if not srcs or source_digest(srcs) != kv.get("source_digest"):
            return None
        return float(kv["dram_bytes_per_step"])
    except (OSError, KeyError, ValueError):
        return None


def timed_replays(graph_list, reps: int, stream):
    """Median microseconds of one replay: `reps` replays (cycling through the
    graphs), each bracketed by events on `stream`."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    with torch.cuda.stream(stream):
        for r, (e0, e1) in enumerate(evs):
            e0.record(stream)
            graph_list[r % len(graph_list)].replay()
            e1.record(stream)
    stream.synchronize()
    return float(np.median([e0.elapsed_time(e1) for e0, e1 in evs])) * 1e3


def run_ours(args):
    import torch

    import mixed_precision_quantized_kvq_b200 as kvq

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist("nccl")
    w = WORKLOADS[args.workload]
    lens0, lens1 = cache_lens(w)
    max_len = int(lens1.max())
    pt = wl.page_table(w, np.maximum(0, lens1 - w.window))
    npages = max(1, int((pt >= 0).sum()))
    signs = torch.from_numpy(wl.rotation_signs(w)).to(dev) if w.rotate_keys else None
    lay = kvq.Layout(w.head_dim, w.num_q_heads, w.num_kv_heads, w.k_bits, w.v_bits, w.k_group,
                     w.v_group, w.page_size, w.window, w.rotate_keys, signs, w.k_per_channel)

    def raw(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    # prefill one cache on the GPU, then clone it until the copies exceed 2x L2
    base = kvq.PagedCache.allocate(lay, torch.from_numpy(pt).to(dev), npages)
    kr, vr, _, _, cu, _ = wl.prefill(w, lens0, with_f32=False)
    glens0 = torch.from_numpy(lens0).to(dev)
    zero = torch.zeros_like(glens0)
    kvq.kvq_quantize_append(lay, base, raw(kr), raw(vr), torch.from_numpy(cu).to(dev), zero,
                            int(lens0.max()))
    del kr, vr
    torch.cuda.synchronize()
    step_bytes = algorithmic_bytes(w, lens1)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    n_copies = max(2, math.ceil(2 * l2 / max(1, step_bytes)) + 1) if args.copies <= 0 else args.copies
    def clone_cache(src):
        return kvq.PagedCache(*[t.clone() if isinstance(t, torch.Tensor) else t
                                for t in (src.k_codes, src.v_codes, src.k_meta, src.v_meta, src.k_win, src.v_win)],
                              src.page_table, npages)

    # The timed steps repeat the append at the same lengths on every copy, which
    # moves the same bytes as a real step; with a window it is not idempotent (the
    # slot that position L-W leaves is the slot token L takes), so the output check
    # below runs one step on an untouched copy of the prefilled cache.
    pristine = clone_cache(base) if not args.no_cpu_baseline else None
    caches = [base]
    for _ in range(n_copies - 1):
        caches.append(clone_cache(base))
    qs, knew, vnew = [], [], []
    for i in range(n_copies):
        qr, _ = wl.query(w, i)
        k1, v1, _, _ = wl.new_tokens(w, i)
        qs.append(raw(qr))
        knew.append(raw(k1))
        vnew.append(raw(v1))
    cu1 = torch.arange(w.batch + 1, dtype=torch.int32, device=dev)
    glens1 = torch.from_numpy(lens1).to(dev)
    wsp = kvq.workspace_for(lay, w.batch, max_len, dev)
    out = torch.empty((w.batch, w.num_q_heads, w.head_dim), dtype=torch.float32, device=dev)
    lse = torch.empty((w.batch, w.num_q_heads), dtype=torch.float32, device=dev)
    scale = 1.0 / math.sqrt(w.head_dim)
    # kernels per step: the append (one launch for one token per sequence; the
    # per-channel layout adds its ring write), then the decode: one persistent
    # kernel, or a split kernel and its combine
    path = kvq.kvq_get_decode_path(lay)
    if w.k_per_channel:
        launches_per_step, decode_kernel = 3, "kvq_decode_attention (per-channel decode kernel: warp-independent tiles, tensor-core scores and weighted values)"
    elif path == kvq.DECODE_TENSOR_CORES:
        launches_per_step, decode_kernel = 2, "kvq_decode_attention (persistent tensor-core kernel, merge fused)"
    else:
        launches_per_step, decode_kernel = 3, "kvq_decode_attention (split-K kernel + combine)"

    def append(i):
        c = caches[i % n_copies]
        kvq.kvq_quantize_append(lay, c, knew[i % n_copies], vnew[i % n_copies], cu1, glens0, 1)

    def decode(i, qq=None):
        c = caches[i % n_copies]
        kvq.kvq_decode_attention(lay, c, qs[i % n_copies] if qq is None else qq, glens1, max_len, scale, out,
                                 lse, wsp)

    def step(i):
        # one call: the append, then the decode, whose start-up overlaps the append
        c = caches[i % n_copies]
        kvq.kvq_append_decode(lay, c, knew[i % n_copies], vnew[i % n_copies], cu1, glens0, 1, qs[i % n_copies],
                              glens1, max_len, scale, out, lse, wsp)

    stream = torch.cuda.Stream(device=dev)
    S = n_copies * max(1, args.graph_rounds)
    with torch.cuda.stream(stream):
        for i in range(2 * n_copies):          # eager warm-up before capture
            step(i)
    stream.synchronize()

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        return g

    g_big = capture(lambda: [step(i) for i in range(S)])
    g_one = [capture(lambda c=c: step(c)) for c in range(n_copies)]
    g_dec = [capture(lambda c=c: decode(c)) for c in range(n_copies)]
    g_app = [capture(lambda c=c: append(c)) for c in range(n_copies)]

    def run_steps(k, start=0):
        """k steps through graph replays; returns the next step index."""
        i = start
        while k > 0:
            if i % n_copies == 0 and k >= S:
                g_big.replay()
                i += S
                k -= S
            else:
                g_one[i % n_copies].replay()
                i += 1
                k -= 1
        return i

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    with torch.cuda.stream(stream):
        nxt = run_steps(args.warmup)
        nxt = (nxt + n_copies - 1) // n_copies * n_copies
    stream.synchronize()
    if dist is not None:
        dist.barrier()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    wall0 = time.time()
    with torch.cuda.stream(stream):
        t_start.record(stream)
        run_steps(args.steps, nxt)
        t_end.record(stream)
    stream.synchronize()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    ms = t_start.elapsed_time(t_end)
    ms_max = reduce_max(dist, ms, dev)
    us_step = ms_max * 1e3 / max(1, args.steps)
    # medians over single-graph replays (each bracketed by events; every replay
    # reads the next cache copy, so each reads HBM)
    reps = max(200, args.median_reps)
    med_step = reduce_max(dist, timed_replays(g_one, reps, stream), dev)
    dec_us = reduce_max(dist, timed_replays(g_dec, reps, stream), dev)
    app_us = reduce_max(dist, timed_replays(g_app, reps, stream), dev)
    wall1 = time.time()

    # e2e through the public API: each step copies its inputs (q, new k, new v
    # packed in one pinned host buffer) to the device in one copy, appends,
    # decodes and reads the output back; captured in a CUDA graph per cache copy
    qn, kn = qs[0].numel() * qs[0].element_size(), knew[0].numel() * knew[0].element_size()
    total = qn + 2 * kn
    hstage = []
    for c in range(n_copies):
        hb = torch.empty(total, dtype=torch.uint8).pin_memory()
        hb[:qn].copy_(qs[c].view(torch.uint8).reshape(-1).cpu())
        hb[qn:qn + kn].copy_(knew[c].view(torch.uint8).reshape(-1).cpu())
        hb[qn + kn:].copy_(vnew[c].view(torch.uint8).reshape(-1).cpu())
        hstage.append(hb)
    dstage = torch.empty(total, dtype=torch.uint8, device=dev)
    dq = dstage[:qn].view(qs[0].dtype).view(qs[0].shape)
    dk = dstage[qn:qn + kn].view(knew[0].dtype).view(knew[0].shape)
    dv = dstage[qn + kn:].view(vnew[0].dtype).view(vnew[0].shape)
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()

    def e2e_step(c):
        dstage.copy_(hstage[c], non_blocking=True)
        kvq.kvq_append_decode(lay, caches[c], dk, dv, cu1, glens0, 1, dq, glens1, max_len, scale, out, lse, wsp)
        hout.copy_(out, non_blocking=True)

    g_e2e = [capture(lambda c=c: e2e_step(c)) for c in range(n_copies)]
    k_e2e = max(1, min(args.steps, args.e2e_steps))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for c in range(n_copies):
            g_e2e[c].replay()
        e0.record(stream)
        for i in range(k_e2e):
            g_e2e[i % n_copies].replay()
        e1.record(stream)
    stream.synchronize()
    e2e_us = reduce_max(dist, e0.elapsed_time(e1) * 1e3 / k_e2e, dev)
    e2e_med = reduce_max(dist, timed_replays(g_e2e, reps, stream), dev)

    sampler.stop()
    clocks = sampler.summary(wall0, wall1)
    peak, peak_kind = measured_hbm_peak()
    achieved = step_bytes / (dec_us * 1e-6) / 1e9
    traffic = profile_traffic(args.workload)
    line = {
        "metric": METRIC, "value": us_step, "unit": "us/step", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": us_step / 1e3, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded; bf16 N(0,1) with key outlier channels)",
        "config": dict(workload_config(w, lens1),
                       l2=f"{n_copies} rotating cache copies ({n_copies * step_bytes / 1e6:.0f} MB of "
                          f"decode reads) > 2x L2 ({l2 / 1e6:.0f} MB)"),
        "hbm_gbs": achieved, "pct_hbm_peak": 100.0 * achieved / peak,
        "median_us": {"step": med_step, "decode_attention": dec_us, "append": app_us, "e2e_step": e2e_med,
                      "replays": reps,
                      "method": "median of single-graph replays, each bracketed by CUDA events on the stream"},
        "breakdown_us": {"append": app_us, "decode_attention": dec_us},
        "algorithmic_bytes_per_step": step_bytes,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic, "kernel": decode_kernel,
                     "duration_us": dec_us,
                     "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)" if peak_kind == "measured"
                     else "fallback 6650 GB/s"},
        "e2e": {"value": e2e_us, "unit": "us/step", "h2d_bytes_per_step": total,
                "d2h_bytes_per_step": out.numel() * out.element_size(),
                "api": "python binding -> C ABI; one H2D copy of the packed step inputs from pinned memory, "
                       "kvq_append_decode (append, then decode) and the D2H read of the output captured in one "
                       "CUDA graph per step"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        # the oracle's first step has the inputs of step 0 on the prefilled cache: compare outputs
        with torch.cuda.stream(stream):
            kvq.kvq_append_decode(lay, pristine, knew[0], vnew[0], cu1, glens0, 1, qs[0], glens1, max_len, scale, out,
                                  lse, wsp)
        stream.synchronize()
        got = out.cpu().numpy()
        us_cpu, cores, sample, ref = oracle_step_timer(w, args.cpu_budget)
        err = np.abs(got.astype(np.float64) - ref)
        lim = 1e-3 + 1e-3 * np.abs(ref)
        line["cpu_baseline"] = {"value": us_cpu, "unit": "us/step", "cores": cores, "kind": "oracle",
                                "sample": sample, "tiny_single_thread_us": oracle_tiny_single_thread(),
                                "oracle_check": {"what": "decode output of the first step (all sequences and "
                                                         "heads) against the fp64 oracle on the same cache",
                                                 "max_abs": float(err.max()),
                                                 "max_rel_ref_gt_1e-2": float((err / np.maximum(np.abs(ref), 1e-30))
                                                                              [np.abs(ref) > 1e-2].max()),
                                                 "within_1e-3_plus_1e-3_rel": bool(np.all(err <= lim))}}
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g_big, g_one, g_dec, g_app, g_e2e
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def prefill_flops(lens, n, d: int, hq: int) -> float:
    """Algorithmic flops of a chunked-prefill attention call: per (query,
    head, visible position) 2d for q.k and 2d for p.v; query i of a chunk of
    n at the end of L positions sees L - n + i + 1 of them."""
    vis = 0
    for L, m in zip(lens, n):
        L, m = int(L), int(m)
        vis += m * (L - m) + m * (m + 1) // 2
    return 4.0 * d * hq * vis


def oracle_prefill_timer(w: wl.Workload, chunk: int):
    """Oracle (fp64, all host threads) on one sequence of the workload:
    quantize its cache, then the chunk's causal attention; returns (seconds,
    threads, sample description)."""
    import oracle
    L = w.seq_len
    w1 = w.with_(batch=1, ragged=None)
    lens = np.array([L], np.int32)
    pt = wl.page_table(w1, np.maximum(0, lens - w1.window))
    c = oracle.Cache(oracle.Layout.from_workload(w1), 1, pt, max(1, int((pt >= 0).sum())))
    kr, vr, _, _, cu, _ = wl.prefill(w1, lens, with_f32=False)
    c.append(kr, vr, oracle.IN_BF16, cu, np.zeros(1, np.int32))
    q, _ = wl.chunk_queries(w1, chunk)
    cu_q = np.array([0, chunk], np.int32)
    t0 = time.perf_counter()
    c.prefill_attention(q, oracle.IN_BF16, cu_q, lens, 1.0 / np.sqrt(w.head_dim))
    dt = time.perf_counter() - t0
    return dt, oracle.num_threads(), f"1 of {w.batch} sequences (chunk {chunk} at the end of {L} positions)"


def run_prefill(args):
    """Chunked-prefill attention (kvq_prefill_attention): every sequence holds
    seq_len positions whose newest `chunk` are the chunk being prefilled; one
    step is one call over the whole batch.  L2 is flushed (a 256 MB write)
    before every timed call; each call is timed with events on its stream."""
    import torch

    import mixed_precision_quantized_kvq_b200 as kvq

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist("nccl")
    w, chunk = PREFILL_WORKLOADS[args.workload]
    B, L = w.batch, w.seq_len
    lens = np.full(B, L, np.int32)
    n = np.full(B, chunk, np.int32)
    pt = wl.page_table(w, np.maximum(0, lens - w.window))
    lay = kvq.Layout(w.head_dim, w.num_q_heads, w.num_kv_heads, w.k_bits, w.v_bits, w.k_group,
                     w.v_group, w.page_size, w.window, False, None)
    cache = kvq.PagedCache.allocate(lay, torch.from_numpy(pt).to(dev), max(1, int((pt >= 0).sum())))

    def raw(a):
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).to(dev)

    kr, vr, _, _, cu, _ = wl.prefill(w, lens, with_f32=False)
    glens = torch.zeros(B, dtype=torch.int32, device=dev)
    kvq.kvq_quantize_append(lay, cache, raw(kr), raw(vr), torch.from_numpy(cu).to(dev), glens, L)
    del kr, vr
    glens.copy_(torch.from_numpy(lens))
    cu_q = torch.from_numpy(np.concatenate([[0], np.cumsum(n)]).astype(np.int32)).to(dev)
    q = raw(wl.chunk_queries(w, int(n.sum()))[0])
    out = torch.empty((int(n.sum()), w.num_q_heads, w.head_dim), dtype=torch.float32, device=dev)
    lse = torch.empty((int(n.sum()), w.num_q_heads), dtype=torch.float32, device=dev)
    scale = 1.0 / np.sqrt(w.head_dim)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]

    def call():
        kvq.kvq_prefill_attention(lay, cache, q, cu_q, glens, chunk, scale, out, lse, stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            flush.fill_(1)
            call()
    stream.synchronize()
    if dist is not None:
        dist.barrier()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    wall0 = time.time()
    with torch.cuda.stream(stream):
        for e0, e1 in evs:
            flush.fill_(1)
            e0.record(stream)
            call()
            e1.record(stream)
    stream.synchronize()
    wall1 = time.time()
    sampler.stop()
    us = float(np.mean([e0.elapsed_time(e1) for e0, e1 in evs])) * 1e3
    us_max = reduce_max(dist, us, dev)

    # e2e: the chunk's queries from pinned host memory, outputs back, every step
    hq_ = q.cpu().pin_memory()
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    dq = torch.empty_like(q)
    k_e2e = max(1, min(args.steps, 20))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(k_e2e):
            dq.copy_(hq_, non_blocking=True)
            kvq.kvq_prefill_attention(lay, cache, dq, cu_q, glens, chunk, scale, out, lse, stream)
            hout.copy_(out, non_blocking=True)
        e1.record(stream)
    stream.synchronize()
    e2e_us = reduce_max(dist, e0.elapsed_time(e1) * 1e3 / k_e2e, dev)

    flops = prefill_flops(lens, n, w.head_dim, w.num_q_heads)
    props = torch.cuda.get_device_properties(dev)
    clocks = sampler.summary(wall0, wall1)
    sm_max = float((clocks or {}).get("sm_max_mhz") or 1965.0)
    achieved = flops / (us * 1e-6) / 1e12
    if prefill_on_tensor_cores(w):
        # bf16 mma.sync with each operand split into (hi, lo): three bf16 products per
        # algorithmic product; reported against the dense bf16 tensor peak
        peak, kind = measured_bf16_peak()
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "traffic": None, "kernel": "kvq_prefill_attention (bf16 tensor cores, operands as bf16 hi/lo "
                                           "pairs: 3 tensor products per algorithmic product)",
                "peak_source": f"{kind} dense bf16 TFLOP/s" + (" (MEASURED_PEAKS.json)" if kind == "measured" else ""),
                "tensor_flops_executed_per_step": 3 * flops}
    else:
        peak = props.multi_processor_count * 128 * 2 * sm_max * 1e6 / 1e12   # fp32 FMA lanes x 2 flops x clock
        roof = {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "traffic": None, "kernel": "kvq_prefill_attention (CUDA cores)",
                "peak_source": f"{props.multi_processor_count} SMs x 128 fp32 lanes x 2 flops x {sm_max:.0f} MHz"}
    line = {
        "metric": PREFILL_METRIC, "value": us_max, "unit": "us/step", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": us_max / 1e3, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded; bf16 N(0,1) with key outlier channels)",
        "config": {"workload": f"{args.workload}: batch {B}, {L} positions, chunk {chunk} (causal), "
                               f"{w.num_q_heads}/{w.num_kv_heads} heads, d{w.head_dim}, K{w.k_bits}V{w.v_bits}, "
                               f"window {w.window}", "l2": "flushed (256 MB write) before every call"},
        "tflops": achieved, "flops_per_step": flops,
        "roofline": roof,
        "e2e": {"value": e2e_us, "unit": "us/step", "h2d_bytes_per_step": q.numel() * q.element_size(),
                "d2h_bytes_per_step": out.numel() * out.element_size(),
                "api": "python binding -> C ABI, eager calls, pinned host buffers"},
        "gpu_launches": args.steps,
        "clocks": clocks,
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        dt, cores, sample = oracle_prefill_timer(w, chunk)
        line["cpu_baseline"] = {"value": dt * 1e6 * B, "unit": "us/step", "cores": cores, "kind": "oracle",
                                "sample": sample + f", scaled x{B} to the batch"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def run_prefill_reference(args):
    """The oracle (as it stands, all host threads) on the chunked-prefill
    workload: each step times one sequence's chunk (cache quantization not
    timed) and scales it to the batch.  Rank 0 only."""
    ws, rank, local = dist_env()
    dist = init_dist("gloo")
    if rank == 0:
        w, chunk = PREFILL_WORKLOADS[args.workload]
        times, cores, sample = [], 1, ""          # no warm-up: the oracle keeps no state between steps
        for _ in range(max(1, args.steps)):
            dt, cores, sample = oracle_prefill_timer(w, chunk)
            times.append(dt * 1e6 * w.batch)
        us = float(np.mean(times))
        line = {"impl": "reference", "metric": PREFILL_METRIC, "value": us, "unit": "us/step", "n_gpus": ws,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": us / 1e3, "higher_is_better": False,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": f"{args.workload}: batch {w.batch}, {w.seq_len} positions, chunk {chunk} "
                                       f"(causal), {w.num_q_heads}/{w.num_kv_heads} heads, d{w.head_dim}, "
                                       f"K{w.k_bits}V{w.v_bits}, window {w.window}"},
                "cpu_baseline": {"value": us, "unit": "us/step", "cores": cores, "kind": "oracle",
                                 "sample": sample + f", scaled x{w.batch} to the batch"},
                "e2e": {"value": us, "unit": "us/step", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + sorted(PREFILL_WORKLOADS), default="llama8b")
    ap.add_argument("--copies", type=int, default=0, help="cache copies to rotate (0 = auto from L2 size)")
    ap.add_argument("--graph-rounds", type=int, default=4)
    ap.add_argument("--e2e-steps", type=int, default=300)
    ap.add_argument("--median-reps", type=int, default=200, help="replays per median (at least 200)")
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--ref-sample-seqs", type=int, default=2)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.workload in PREFILL_WORKLOADS:
        if args.impl == "reference":
            run_prefill_reference(args)
        else:
            run_prefill(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
