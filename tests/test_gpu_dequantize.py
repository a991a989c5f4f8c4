"""GPU parity of kvq_dequantize (the check path: "dequantization into
temporary storage", "Kuantisasi KV cache ...", section "Pertumbuhan cache
mengubah trade pada serving") against the oracle's reconstruction, bit for
bit: head_dim 128 with per-token groups, with and without the bf16 window,
with keys in the rotated domain, and on the full 8B-layer and rotation
workloads."""
import numpy as np
import pytest
import torch

import mixed_precision_quantized_kvq_b200 as kvq
import oracle
import workloads as wl
from gpu_harness import Pair, torch_raw

pytestmark = pytest.mark.gpu


def small(**kw):
    base = dict(name="small", batch=4, num_q_heads=8, num_kv_heads=2, head_dim=128, seq_len=0,
                k_bits=4, v_bits=2, k_group=32, v_group=128, window=0, ragged=(1, 700),
                shuffle_pages=True, outliers=("random", 4, 10.0), seed=11)
    base.update(kw)
    return wl.Workload(**base)


def rotated_pair(w, lens, steps=0):
    """A pair whose oracle side quantizes the library's rotated keys (the
    rotation itself agrees with the oracle's fp64 product to round-off; the
    codes are compared from the rotated fp32 keys on).  Positions that stay
    in the bf16 window keep their unrotated keys."""
    pair = Pair(w, lens, steps=steps)
    kr, vr, kf, _, cu, _ = wl.prefill(w, lens)
    rot = torch.empty(kr.shape, dtype=torch.float32, device="cuda")
    kvq.kvq_rotate_keys(pair.glay, torch_raw(kr), rot)
    rot = rot.cpu().numpy()
    # rotated rows where the position ends up quantized, raw rows in the window
    rows = kf.astype(np.float32).copy()
    for b in range(w.batch):
        nq = max(0, int(lens[b]) - w.window)
        rows[cu[b]:cu[b] + nq] = rot[cu[b]:cu[b] + nq]
    olay = oracle.Layout.from_workload(w.with_(rotate_keys=False))
    pair.ocache = oracle.Cache(olay, w.batch, pair.pt, pair.num_pages)
    pair.lens[:] = 0
    pair.glens.zero_()
    pair.append(kr, vr, cu, oracle_k=np.ascontiguousarray(rows), oracle_dtype=oracle.IN_F32)
    return pair


@pytest.mark.parametrize("window", [0, 100, 128, 5000])
@pytest.mark.parametrize("kb,vb", [(4, 2), (8, 8), (1, 2), (2, 4)])
def test_dequantize_d128(kb, vb, window):
    w = small(k_bits=kb, v_bits=vb, window=window)
    lens = wl.lengths(w)
    lens[1] = 0                          # an empty sequence is left untouched
    pair = Pair(w, lens)
    pair.prefill(with_f32=False)
    pair.compare_cache()
    pair.check_dequantize()
    pair.check_dequantize(max_len=int(lens.max()) + 37)   # room past every length


@pytest.mark.parametrize("window", [0, 64])
def test_dequantize_rotated_keys(window):
    """Keys come back in the rotated domain (code*scale+zero of the rotated
    row); window keys stay unrotated bf16."""
    w = small(rotate_keys=True, window=window, outliers=("student_t", 4, 10.0, 3.0))
    pair = rotated_pair(w, wl.lengths(w))
    pair.compare_cache()
    pair.check_dequantize()


def test_dequantize_after_decode_appends():
    """Tokens that left the window through single-token appends reconstruct
    like the prefilled ones."""
    w = small(window=48, ragged=(40, 300))
    lens = wl.lengths(w)
    pair = Pair(w, lens, steps=6)
    pair.prefill(with_f32=False)
    for s in range(6):
        k1, v1, _, _ = wl.new_tokens(w, s)
        pair.append(k1, v1, np.arange(w.batch + 1, dtype=np.int32))
    pair.compare_cache()
    pair.check_dequantize()


def test_dequantize_llama8b_full():
    """The 8B-layer workload at full size (B16, 32/8 heads, d128, 4096
    tokens, K4 g32 / V2 g128, W128) after two decode appends."""
    w = wl.LLAMA8B
    pair = Pair(w, wl.lengths(w), steps=2)
    pair.prefill(with_f32=False)
    for s in range(2):
        k1, v1, _, _ = wl.new_tokens(w, s)
        pair.append(k1, v1, np.arange(w.batch + 1, dtype=np.int32))
    pair.check_dequantize()


def test_dequantize_rotation_full():
    """The key-rotation workload at full size (B32, d128, 8192 tokens, K4V2)."""
    w = wl.ROTATION
    pair = rotated_pair(w, wl.lengths(w))
    pair.check_dequantize()
