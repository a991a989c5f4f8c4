"""kvq_append_decode (one decode step: append, then decode attention) against
the two calls it stands for, kvq_quantize_append then kvq_decode_attention,
on identical caches: cache bytes and attention outputs bit for bit.  Covers
the overlapped launch (one-launch append, persistent tensor-core decode) and
the cases that run the two calls one after the other (appends of more than
eight tokens, the CUDA-core decode path, per-channel key groups).  The
separate calls are checked against the oracle by the parity tests."""
import math

import numpy as np
import pytest
import torch

import mixed_precision_quantized_kvq_b200 as kvq
import workloads as wl
from gpu_harness import Pair, torch_raw

pytestmark = pytest.mark.gpu

CACHE_FIELDS = ("k_codes", "v_codes", "k_meta", "v_meta", "k_win", "v_win")


def small(**kw):
    base = dict(name="small", batch=5, num_q_heads=8, num_kv_heads=2, head_dim=128, seq_len=0,
                k_bits=4, v_bits=2, k_group=32, v_group=128, window=0, ragged=(1, 700),
                shuffle_pages=True, outliers=("random", 4, 10.0), seed=21)
    base.update(kw)
    return wl.Workload(**base)


def clone_cache(c: kvq.PagedCache) -> kvq.PagedCache:
    f = lambda t: None if t is None else t.clone()
    return kvq.PagedCache(f(c.k_codes), f(c.v_codes), f(c.k_meta), f(c.v_meta), f(c.k_win), f(c.v_win),
                          c.page_table, c.num_pages)


def run_step(w, n_new, path=kvq.DECODE_AUTO, steps=2):
    lens0 = wl.lengths(w)
    lens0[1] = 0                                   # an empty sequence that starts filling
    pair = Pair(w, lens0, steps=steps * n_new + 8)
    pair.prefill(with_f32=False)
    sep = pair.gcache
    comb = clone_cache(sep)
    lay = pair.glay
    B, Hq, d = w.batch, w.num_q_heads, w.head_dim
    glens = torch.from_numpy(lens0).cuda()
    cu = torch.arange(0, (B + 1) * n_new, n_new, dtype=torch.int32, device="cuda")
    kvq.kvq_set_decode_path(path)
    try:
        for s in range(steps):
            rows = [wl.new_tokens(w, 100 * s + i) for i in range(n_new)]
            k = np.stack([r[0] for r in rows], 1).reshape(B * n_new, w.num_kv_heads, d)
            v = np.stack([r[1] for r in rows], 1).reshape(B * n_new, w.num_kv_heads, d)
            kt, vt = torch_raw(k), torch_raw(v)
            q = torch_raw(wl.query(w, s)[0])
            lens1 = glens + n_new
            max_len = int(lens1.max())
            ws = kvq.workspace_for(lay, B, max_len, "cuda")
            outs = []
            for cache, combined in ((sep, False), (comb, True)):
                out = torch.full((B, Hq, d), 7.0, device="cuda")
                lse = torch.full((B, Hq), 7.0, device="cuda")
                if combined:
                    kvq.kvq_append_decode(lay, cache, kt, vt, cu, glens, n_new, q, lens1, max_len,
                                          1 / math.sqrt(d), out, lse, ws)
                else:
                    kvq.kvq_quantize_append(lay, cache, kt, vt, cu, glens, n_new)
                    kvq.kvq_decode_attention(lay, cache, q, lens1, max_len, 1 / math.sqrt(d), out, lse, ws)
                outs.append((out, lse))
            torch.cuda.synchronize()
            for name in CACHE_FIELDS:
                a, b = getattr(sep, name), getattr(comb, name)
                assert (a is None) == (b is None)
                if a is not None:
                    assert torch.equal(a, b), f"{name} differs after step {s}"
            assert torch.equal(outs[0][0], outs[1][0]), f"out differs after step {s}"
            assert torch.equal(outs[0][1], outs[1][1]), f"lse differs after step {s}"
            assert torch.isfinite(outs[1][0]).all()
            glens = lens1
    finally:
        kvq.kvq_set_decode_path(kvq.DECODE_AUTO)


@pytest.mark.parametrize("window,n_new", [(0, 1), (64, 1), (128, 3), (16, 8)])
def test_overlapped_step_matches_separate_calls(window, n_new):
    run_step(small(window=window), n_new)


@pytest.mark.parametrize("kb,vb", [(8, 8), (2, 4), (1, 2)])
def test_overlapped_step_other_bit_widths(kb, vb):
    run_step(small(k_bits=kb, v_bits=vb, window=32), 1)


def test_rotated_keys_step():
    run_step(small(rotate_keys=True, window=40, outliers=("student_t", 4, 10.0, 3.0)), 1)


def test_long_append_runs_the_calls_in_turn():
    """More new tokens than the one-launch append takes."""
    run_step(small(window=64), 12)


def test_cuda_core_path_step():
    run_step(small(window=64), 1, path=kvq.DECODE_CUDA_CORES)


def test_per_channel_step():
    run_step(small(window=64, k_per_channel=True, k_group=32), 1)


def test_full_8b_layer_step():
    """The bench's step at full size: B16, 32/8 heads, d128, 4096 tokens, K4V2, W128."""
    run_step(wl.LLAMA8B, 1, steps=2)
