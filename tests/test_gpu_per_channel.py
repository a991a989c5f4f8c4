"""GPU parity of per-channel key groups (key groups of k_group positions of
one channel, the bf16 window as residual buffer) against the oracle.

Cache bytes (codes, metadata, ring) must be bit-identical to the oracle's
after a prefill, after single-token decode steps and after a chunk that
completes several groups; dequantize must return the oracle's values;
decode and chunked-prefill attention must agree with the fp64 oracle within
1e-3 + 1e-3 * |ref|.
"""
import numpy as np
import pytest
import torch

import mixed_precision_quantized_kvq_b200 as kvq
import workloads as wl
from gpu_harness import Pair, check_close, in_code, torch_raw

pytestmark = pytest.mark.gpu


def pc(**kw):
    base = dict(name="per_channel", batch=4, num_q_heads=16, num_kv_heads=4, head_dim=128, seq_len=0,
                k_bits=4, v_bits=2, k_group=64, v_group=128, window=32, k_per_channel=True,
                ragged=(1, 600), shuffle_pages=True, outliers=("random", 4, 10.0), seed=29)
    base.update(kw)
    return wl.Workload(**base)


def _rows(w, start, n):
    ks, vs = [], []
    for b in range(w.batch):
        if n[b]:
            kr, vr, _, _ = wl.seq_kv(w, b, int(n[b]), start=int(start[b]))
            ks.append(kr)
            vs.append(vr)
    return np.concatenate(ks), np.concatenate(vs)


def _prefill_check(pair):
    w = pair.w
    n = np.minimum(pair.lens, 50).astype(np.int32)
    cu_q = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    q, _ = wl.chunk_queries(w, int(cu_q[-1]), step=3)
    sc = 1.0 / np.sqrt(w.head_dim)
    out, lse = kvq.prefill_attention(pair.glay, pair.gcache, torch_raw(q), torch.from_numpy(cu_q).cuda(),
                                     pair.glens, int(n.max()), sc)
    ref, ref_lse = pair.ocache.prefill_attention(q, in_code(w), cu_q, pair.lens, sc)
    check_close(out.cpu().numpy(), ref, "prefill out")
    check_close(lse.cpu().numpy(), ref_lse, "prefill lse")


CASES = {
    "k4v2_g64_w32": dict(),
    "k4v2_g32_w0": dict(k_group=32, window=0),
    "k2v2_g16_w8": dict(k_bits=2, k_group=16, window=8),
    "k1v1_g16_w8_d64": dict(head_dim=64, k_bits=1, v_bits=1, k_group=16, v_group=64, window=8),
    "k8v4_g32_w128_f32": dict(k_bits=8, v_bits=4, k_group=32, window=128, in_dtype=wl.DT_F32),
    # five and eight query heads per kv-head (the decode kernel's 8-head build), smaller value groups
    "k4v2_g64_w64_gqa5_vg64": dict(num_q_heads=20, v_group=64, window=64),
    "k4v4_g16_w0_gqa8_vg32": dict(num_q_heads=32, v_bits=4, k_group=16, v_group=32, window=0),
}


@pytest.mark.parametrize("name", list(CASES))
def test_append_decode_prefill(name):
    w = pc(**CASES[name])
    lens0 = wl.lengths(w)
    lens0[0] = 0
    steps, chunk = 24, 130
    pair = Pair(w, lens0, steps=steps + chunk)
    pair.prefill(with_f32=False)
    pair.compare_cache()
    pair.check_decode(step=0)
    ones = np.arange(w.batch + 1, dtype=np.int32)
    for s in range(steps):
        k, v = _rows(w, pair.lens, np.ones(w.batch, np.int32))
        pair.append(k, v, ones)
        if s % 6 == 5:
            pair.compare_cache()
            pair.check_decode(step=s)
    n = np.array([chunk, 1, 65, 0][:w.batch], np.int32)
    k, v = _rows(w, pair.lens, n)
    pair.append(k, v, np.concatenate([[0], np.cumsum(n)]).astype(np.int32))
    pair.compare_cache()
    pair.check_decode(step=99)
    _prefill_check(pair)
    kh, vh = pair.dequantize()
    okh, ovh = pair.ocache.dequantize(pair.lens, int(pair.lens.max()))
    for b in range(w.batch):
        L = int(pair.lens[b])
        np.testing.assert_array_equal(kh[b, :, :L], okh[b, :, :L])
        np.testing.assert_array_equal(vh[b, :, :L], ovh[b, :, :L])


def test_empty_sequences_and_static_scratch_entry():
    """An empty sequence gets out = 0, lse = -inf; the static-scratch entry
    point needs no scratch for this layout and gives the same result."""
    w = pc(window=16)
    lens = wl.lengths(w)
    lens[1] = 0
    pair = Pair(w, lens)
    pair.prefill(with_f32=False)
    out, ref = pair.check_decode(step=5)
    q = torch_raw(wl.query(w, 5)[0])
    sc = 1.0 / np.sqrt(w.head_dim)
    o2 = torch.empty((w.batch, w.num_q_heads, w.head_dim), device="cuda")
    l2 = torch.empty((w.batch, w.num_q_heads), device="cuda")
    kvq.kvq_decode_attention_static_scratch(pair.glay, pair.gcache, q, pair.glens, int(lens.max()), sc, o2, l2)
    torch.cuda.synchronize()
    assert torch.equal(o2.cpu(), torch.from_numpy(np.asarray(out, np.float32)))
    assert torch.all(o2[1] == 0) and torch.all(torch.isinf(l2[1]))


def test_split_pairs():
    """Few (sequence, kv-head) pairs with long sequences: each pair's tiles
    are split between CTAs that merge through the workspace (the last CTA to
    finish merges every split in split order).  Against the oracle, with an
    empty sequence; the static-scratch entry point gives the same bits; the
    call without a workspace (one CTA per pair) agrees within tolerance.  The
    third sequence holds two tiles, so most of its splits have none and store
    empty parts."""
    w = pc(batch=3, num_kv_heads=2, num_q_heads=8, ragged=(2500, 4200), window=64, k_group=64, v_group=64)
    lens = wl.lengths(w)
    lens[1] = 0
    lens[0] = max(int(lens[0]), 3000)
    lens[2] = 100
    pair = Pair(w, lens)
    pair.prefill(with_f32=False)
    max_len = int(lens.max())
    assert kvq.kvq_decode_workspace_bytes(pair.glay, w.batch, max_len) > 0   # the split is taken
    out, ref = pair.check_decode(step=2)
    q = torch_raw(wl.query(w, 2)[0])
    sc = 1.0 / np.sqrt(w.head_dim)
    o2 = torch.empty((w.batch, w.num_q_heads, w.head_dim), device="cuda")
    l2 = torch.empty((w.batch, w.num_q_heads), device="cuda")
    kvq.kvq_decode_attention_static_scratch(pair.glay, pair.gcache, q, pair.glens, max_len, sc, o2, l2)
    o3 = torch.empty_like(o2)
    l3 = torch.empty_like(l2)
    kvq.kvq_decode_attention(pair.glay, pair.gcache, q, pair.glens, max_len, sc, o3, l3, None)
    torch.cuda.synchronize()
    assert torch.equal(o2.cpu(), torch.from_numpy(np.asarray(out, np.float32)))
    check_close(o3.cpu().numpy(), ref, "out without a workspace")
    assert torch.all(o2[1] == 0) and torch.all(torch.isinf(l2[1]))
