"""Pins of the oracle's paged cache: layout plumbing, the recent-token bf16
window, decode attention with GQA and ragged lengths, key-only rotation, and
the memory figures.

"Kuantisasi KV cache mengganggu attention ...", section "Pertumbuhan cache
mengubah trade pada serving": recent tokens stay at higher precision, older
blocks are quantized; memory counts payload plus metadata.  "Quantize What
Counts ..." (Belangrijkste Bijdragen): K4V2 vs K4V4 saves 25% of the cache.
"""
import os

import numpy as np
import pytest
import scipy.linalg
import scipy.special

import oracle
import workloads as wl

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    out = {}
    for line in open(os.path.join(GOLD, name)):
        line = line.strip()
        if line and not line.startswith("#") and "=" in line:
            k, v = line.split("=")
            out[k.strip()] = float(v)
    return out


def test_memory_figures_against_pages():
    g = _gold("memory_k4v2_vs_k4v4.txt")
    k4v2 = oracle.page_bytes(oracle.Layout(128, 32, 8, 4, 2, 32, 128, 64, 0))
    k4v4 = oracle.page_bytes(oracle.Layout(128, 32, 8, 4, 4, 32, 128, 64, 0))
    per = 8 * 64  # kv-heads x tokens per page
    payload = lambda pb: pb[0] + pb[2]
    assert 1 - payload(k4v2) / payload(k4v4) == g["payload_reduction_k4v2_vs_k4v4"]
    assert sum(k4v2) / per == g["token_head_bytes_k4v2_g32_g128_d128"]
    assert sum(k4v4) / per == g["token_head_bytes_k4v4_g32_g128_d128"]


def test_packing_fixture():
    for line in open(os.path.join(GOLD, "packing_examples.txt")):
        if line.startswith("#") or not line.strip():
            continue
        bits, codes, packed = [p.strip() for p in line.split(":")]
        got = oracle.pack(np.array([int(c) for c in codes.split()]), int(bits))
        assert got.tobytes() == bytes(int(b, 16) for b in packed.split())


SMALL = wl.Workload(name="small", batch=3, num_q_heads=6, num_kv_heads=2, head_dim=64,
                    seq_len=0, k_bits=4, v_bits=2, k_group=32, v_group=64, window=16,
                    ragged=(1, 200), shuffle_pages=True, outliers=("random", 2, 10.0), seed=3)


def _build(w, lens, capacity=None, signs=None):
    cap = capacity if capacity is not None else lens
    pt = wl.page_table(w, cap)
    npages = int((pt >= 0).sum())
    return oracle.Cache(oracle.Layout.from_workload(w, signs), w.batch, pt, npages)


def _prefill(w, lens, cache):
    kr, vr, kf, vf, cu, _ = wl.prefill(w, lens)
    dt = oracle.IN_BF16 if w.in_dtype == wl.DT_BF16 else oracle.IN_F32
    cache.append(kr, vr, dt, cu, np.zeros(w.batch, np.int32))
    return kf, vf, cu


@pytest.mark.parametrize("window", [0, 16, 1000])
def test_prefill_plumbing_matches_group_quantizer(window):
    w = SMALL.with_(window=window)
    lens = wl.lengths(w)
    lens[1] = 0                                         # an empty sequence
    c = _build(w, lens)
    kf, vf, cu = _prefill(w, lens, c)
    kh, vh = c.dequantize(lens, int(lens.max()))
    for b in range(w.batch):
        L = int(lens[b])
        for h in range(w.num_kv_heads):
            k = kf[cu[b]:cu[b + 1], h]
            v = vf[cu[b]:cu[b + 1], h]
            nq = max(0, L - window)
            if nq:
                s, z, cc = oracle.quantize_rows(k[:nq], w.k_group, w.k_bits)
                np.testing.assert_array_equal(kh[b, h, :nq],
                                              oracle.dequantize_rows(cc, s, z, w.k_group))
                s, z, cc = oracle.quantize_rows(v[:nq], w.v_group, w.v_bits)
                np.testing.assert_array_equal(vh[b, h, :nq],
                                              oracle.dequantize_rows(cc, s, z, w.v_group))
            np.testing.assert_array_equal(kh[b, h, nq:L], k[nq:])       # bf16 kept as-is
            np.testing.assert_array_equal(vh[b, h, nq:L], v[nq:])


def test_incremental_append_equals_one_shot():
    """Quantizing a token does not depend on when it leaves the window."""
    w = SMALL
    lens = wl.lengths(w)
    kr, vr, kf, vf, cu, _ = wl.prefill(w, lens)
    one = _build(w, lens)
    one.append(kr, vr, oracle.IN_BF16, cu, np.zeros(w.batch, np.int32))
    inc = _build(w, lens)
    r = np.random.default_rng(9)
    done = np.zeros(w.batch, np.int32)
    while np.any(done < lens):
        n = np.minimum(r.integers(0, 40, w.batch), lens - done).astype(np.int32)
        rows_k, rows_v, cun = [], [], [0]
        for b in range(w.batch):
            rows_k.append(kr[cu[b] + done[b]: cu[b] + done[b] + n[b]])
            rows_v.append(vr[cu[b] + done[b]: cu[b] + done[b] + n[b]])
            cun.append(cun[-1] + int(n[b]))
        inc.append(np.concatenate(rows_k), np.concatenate(rows_v), oracle.IN_BF16,
                   np.array(cun, np.int32), done.copy())
        done = done + n
    for name in ("k_codes", "k_meta", "v_codes", "v_meta", "k_win", "v_win"):
        np.testing.assert_array_equal(getattr(inc, name), getattr(one, name), err_msg=name)


def _expand(arr, g):
    return np.repeat(arr, g, axis=1)


def test_all_window_is_exact_attention():
    """16-bit storage (E_K = E_V = 0) reproduces exact attention."""
    w = SMALL.with_(window=4096)
    lens = wl.lengths(w)
    c = _build(w, lens)
    kf, vf, cu = _prefill(w, lens, c)
    qr, qf = wl.query(w)
    out, lse = c.decode_attention(qr, oracle.IN_BF16, lens, 1 / np.sqrt(w.head_dim))
    g = w.gqa
    for b in range(w.batch):
        for hq in range(w.num_q_heads):
            K = kf[cu[b]:cu[b + 1], hq // g].astype(np.float64)
            V = vf[cu[b]:cu[b + 1], hq // g].astype(np.float64)
            s = K @ qf[b, hq].astype(np.float64) / np.sqrt(w.head_dim)
            np.testing.assert_allclose(out[b, hq], scipy.special.softmax(s) @ V, rtol=1e-11, atol=1e-12)
            assert abs(lse[b, hq] - scipy.special.logsumexp(s)) < 1e-10


@pytest.mark.parametrize("rotate", [False, True])
def test_decode_attention_on_reconstructed_cache(rotate):
    w = SMALL.with_(rotate_keys=rotate)
    lens = wl.lengths(w)
    lens[2] = 0
    signs = wl.rotation_signs(w) if rotate else None
    c = _build(w, lens, signs=signs)
    kf, vf, cu = _prefill(w, lens, c)
    kh, vh = c.dequantize(lens, int(lens.max()))
    qr, qf = wl.query(w)
    sc = 1 / np.sqrt(w.head_dim)
    out, lse = c.decode_attention(qr, oracle.IN_BF16, lens, sc)
    g = w.gqa
    H = scipy.linalg.hadamard(w.head_dim) / np.sqrt(w.head_dim)
    for b in range(w.batch):
        L = int(lens[b])
        nq = max(0, L - w.window)
        for hq in range(w.num_q_heads):
            q = qf[b, hq].astype(np.float64)
            K = kh[b, hq // g, :L].astype(np.float64)
            V = vh[b, hq // g, :L].astype(np.float64)
            if L == 0:
                assert np.all(out[b, hq] == 0) and lse[b, hq] == -np.inf
                continue
            s = K @ q
            if rotate:
                s[:nq] = K[:nq] @ ((q * signs) @ H)
            s *= sc
            np.testing.assert_allclose(out[b, hq], scipy.special.softmax(s) @ V, rtol=1e-10, atol=1e-11)
            assert abs(lse[b, hq] - scipy.special.logsumexp(s)) < 1e-9
        if rotate and nq:
            for h in range(w.num_kv_heads):
                kr = oracle.rotate(kf[cu[b]:cu[b] + nq, h], signs)
                s_, z_, c_ = oracle.quantize_rows(kr, w.k_group, w.k_bits)
                np.testing.assert_array_equal(kh[b, h, :nq], oracle.dequantize_rows(c_, s_, z_, w.k_group))


def test_fp32_inputs_enter_window_rounded_to_bf16():
    w = SMALL.with_(in_dtype=wl.DT_F32, window=8)
    lens = np.array([20, 5, 9], np.int32)
    c = _build(w, lens)
    kf, vf, cu = _prefill(w, lens, c)
    kh, _ = c.dequantize(lens, 20)
    want = wl.bf16_to_f32(oracle.f32_to_bf16(kf[cu[0] + 12:cu[0] + 20, 0].ravel()))
    np.testing.assert_array_equal(kh[0, 0, 12:20].ravel(), want)


def test_chunked_code_positions_hand_derived():
    """Storage format: key rows and value channel runs over 16 bytes are kept
    as 16-byte chunks, chunk-major inside a (page, kv-head) block.  K4 at
    head_dim 128: channel 40 of token slot 5 is nibble 0 of row byte 20 =
    chunk 1, byte 4 -> block offset 1*(64*16) + 5*16 + 4 = 1108.  V4: token
    slot 37 of channel 9 is the high nibble of run byte 18 = chunk 1, byte 2
    -> block offset 1*(128*16) + 9*16 + 2 = 2194."""
    d = 128
    lay = oracle.Layout(d, 1, 1, 4, 4, 32, 128, 64, 0)
    pt = np.zeros((1, 1), np.int32)
    c = oracle.Cache(lay, 1, pt, 1)
    # on-grid values: zero 0, scale 1 -> code == value
    k = np.zeros((64, 1, d), np.float32)
    v = np.zeros((64, 1, d), np.float32)
    k[:, :, 127] = 15.0                      # fixes every key group's range
    for g0 in range(0, d, 32):
        k[:, :, g0 + 31] = 15.0
    v[:, :, 127] = 15.0
    k[5, 0, 40] = 9.0
    v[37, 0, 9] = 6.0
    c.append(k, v, oracle.IN_F32, np.array([0, 64], np.int32), np.zeros(1, np.int32))
    kb = c.k_codes.ravel()
    vb = c.v_codes.ravel()
    assert kb[1108] & 0x0F == 9
    assert (vb[2194] >> 4) == 6
    assert kb[1108 - 16] & 0x0F == 0         # same byte of token slot 4
