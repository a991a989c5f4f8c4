"""Host-side logic of the benchmark (CPU only): byte accounting, the
max-over-ranks reduction with two gloo ranks, and the reference arm's JSON
line, alone and under torchrun with two ranks."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_algorithmic_bytes_hand_derived():
    # 116 B per quantized token-head (64 + 16 + 32 + 4), 512 B per bf16 window token-head
    assert bench.algorithmic_bytes(wl.LLAMA8B, [4096] * 16) == 16 * 8 * (3968 * 116 + 128 * 512)
    assert bench.algorithmic_bytes(wl.LLAMA8B, [4096] * 16) == 67_305_472
    assert bench.algorithmic_bytes(wl.SWEEP, [16384] * 8) == 121_634_816
    assert bench.algorithmic_bytes(wl.ROTATION, [8192] * 32) == 243_269_632
    k8v8 = wl.SWEEP.with_(k_bits=8, v_bits=8)
    assert bench.algorithmic_bytes(k8v8, [16384] * 8) == 8 * 8 * 16384 * (128 + 16 + 128 + 4)
    assert bench.algorithmic_bytes(wl.LLAMA8B, [100]) == 8 * 100 * 512
    assert bench.algorithmic_bytes(wl.LLAMA8B, [0]) == 0


def test_cache_lens():
    l0, l1 = bench.cache_lens(wl.LLAMA8B)
    assert np.all(l1 == 4096) and np.all(l0 == 4095)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE="2", RANK=str(rank),
                      LOCAL_RANK=str(rank))
    dist = bench.init_dist("gloo")
    v = bench.reduce_max(dist, float(rank + 1) * 1.5)
    q.put((rank, v))
    dist.barrier()
    dist.destroy_process_group()


def test_reduce_max_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == {0: 3.0, 1: 3.0}


REQUIRED = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
            "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"}


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "2", "--warmup", "3"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert REQUIRED <= set(d)
    assert d["impl"] == "reference" and d["unit"] == "us/step" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_two_ranks_prints_once():
    port = _free_port()
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
                        "--master-addr", "127.0.0.1", "--master-port", str(port),
                        os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--gpus", "2", "--steps", "2", "--warmup", "3"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    assert json.loads(lines[0])["n_gpus"] == 2


def test_algorithmic_bytes_per_channel_counts_whole_groups():
    """With key groups along positions the pages hold whole groups only; the
    rest of the sequence is read from the bf16 ring."""
    import bench
    import workloads as wl
    w = bench.WORKLOADS["per_channel_llama8b"]
    d, H = w.head_dim, w.num_kv_heads
    t = d * 4 // 8 + 4 * d // 64 + d * 2 // 8 + 4 * d // 64          # 64 + 8 + 32 + 8 = 112
    assert t == 112
    for L in (0, 100, 128, 191, 192, 193, 4096):
        q = max(0, L - 128) // 64 * 64
        assert bench.algorithmic_bytes(w, [L]) == (q * t + (L - q) * 4 * d) * H
    assert bench.algorithmic_bytes(wl.LLAMA8B, [4096]) == (3968 * 116 + 128 * 512) * 8


def test_tiny_single_thread_oracle_timer_restores_threads():
    import bench
    import oracle
    before = oracle.num_threads()
    us = bench.oracle_tiny_single_thread(steps=3)
    assert us > 0 and oracle.num_threads() == before
