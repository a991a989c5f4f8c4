"""Pins of the oracle's per-channel key grouping (key groups of k_group
consecutive positions of one channel, the bf16 window as residual buffer).

"Kuantisasi KV cache mengganggu attention ...", section "Granularitas
kuantisasi menentukan nilai yang berbagi scale": the grouping axis may run
along token positions, channels, heads or blocks; fewer, larger groups need
less metadata.  "Kuantisasi on Nalar" (teaser): outliers set the scale of
the whole group, so a group along positions keeps an outlier channel's
range away from the other channels.  Section "Pertumbuhan cache ...":
recent tokens stay in higher precision; here a key group waits in the bf16
ring until it is complete and out of the W newest positions.
"""
import os

import numpy as np
import pytest
import scipy.special

import oracle
import workloads as wl

GOLD = os.path.join(os.path.dirname(__file__), "golden")

PC = wl.Workload(name="per_channel", batch=3, num_q_heads=8, num_kv_heads=2, head_dim=64, seq_len=0,
                 k_bits=4, v_bits=2, k_group=32, v_group=64, window=16, k_per_channel=True,
                 ragged=(1, 300), shuffle_pages=True, outliers=("random", 2, 10.0), seed=13)


def _cache(w, lens):
    pt = wl.page_table(w, np.maximum(0, np.asarray(lens) - w.window))
    return oracle.Cache(oracle.Layout.from_workload(w), w.batch, pt, max(1, int((pt >= 0).sum())))


def _paged(L, W, G):
    """Positions in pages: complete key groups that left the W newest positions."""
    q = max(0, L - W)
    return q - q % G


def test_memory_figures():
    g = {}
    for line in open(os.path.join(GOLD, "memory_per_channel_keys.txt")):
        if "=" in line and not line.startswith("#"):
            k, v = line.split("=")
            g[k.strip()] = float(v)
    per = 8 * 64
    for kb, G, key in ((4, 64, "token_head_bytes_k4_pc64_v2_g128_d128"),
                       (4, 32, "token_head_bytes_k4_pc32_v2_g128_d128"),
                       (2, 64, "token_head_bytes_k2_pc64_v2_g128_d128")):
        lay = oracle.Layout(128, 32, 8, kb, 2, G, 128, 64, 0, k_per_channel=True)
        assert sum(oracle.page_bytes(lay)) / per == g[key]


@pytest.mark.parametrize("window", [0, 16, 40])
@pytest.mark.parametrize("G", [16, 32, 64])
def test_groups_run_along_positions(window, G):
    """Each page key group of a channel is the group quantizer applied to
    that channel's G positions; values keep per-token groups; exactly the
    positions from kg*floor((L-W)/kg) on are kept as bf16."""
    w = PC.with_(window=window, k_group=G)
    lens = wl.lengths(w)
    lens[0] = 0
    c = _cache(w, lens)
    kr, vr, kf, vf, cu, _ = wl.prefill(w, lens)
    c.append(kr, vr, oracle.IN_BF16, cu, np.zeros(w.batch, np.int32))
    kh, vh = c.dequantize(lens, max(1, int(lens.max())))
    for b in range(w.batch):
        L = int(lens[b])
        Q = _paged(L, window, G)
        for h in range(w.num_kv_heads):
            k = kf[cu[b]:cu[b + 1], h]
            v = vf[cu[b]:cu[b + 1], h]
            for g0 in range(0, Q, G):
                blockT = np.ascontiguousarray(k[g0:g0 + G].T)          # [d][G]: one row per channel
                s, z, cc = oracle.quantize_rows(blockT, G, w.k_bits)
                np.testing.assert_array_equal(kh[b, h, g0:g0 + G], oracle.dequantize_rows(cc, s, z, G).T)
            if Q:
                s, z, cc = oracle.quantize_rows(v[:Q], w.v_group, w.v_bits)
                np.testing.assert_array_equal(vh[b, h, :Q], oracle.dequantize_rows(cc, s, z, w.v_group))
            np.testing.assert_array_equal(kh[b, h, Q:L], k[Q:])
            np.testing.assert_array_equal(vh[b, h, Q:L], v[Q:])


def test_incremental_appends_equal_one_shot():
    """Whether positions arrive one by one or all at once, the same groups
    are quantized from the same values."""
    w = PC
    lens = wl.lengths(w)
    kr, vr, _, _, cu, _ = wl.prefill(w, lens)
    one = _cache(w, lens)
    one.append(kr, vr, oracle.IN_BF16, cu, np.zeros(w.batch, np.int32))
    inc = _cache(w, lens)
    r = np.random.default_rng(4)
    done = np.zeros(w.batch, np.int32)
    while np.any(done < lens):
        n = np.minimum(r.choice([0, 1, 1, 2, 7, 33], w.batch), lens - done).astype(np.int32)
        rows_k, rows_v, cun = [], [], [0]
        for b in range(w.batch):
            rows_k.append(kr[cu[b] + done[b]: cu[b] + done[b] + n[b]])
            rows_v.append(vr[cu[b] + done[b]: cu[b] + done[b] + n[b]])
            cun.append(cun[-1] + int(n[b]))
        inc.append(np.concatenate(rows_k), np.concatenate(rows_v), oracle.IN_BF16,
                   np.array(cun, np.int32), done.copy())
        done = done + n
    for name in ("k_codes", "k_meta", "v_codes", "v_meta"):
        np.testing.assert_array_equal(getattr(inc, name), getattr(one, name), err_msg=name)
    kh1, vh1 = one.dequantize(lens, int(lens.max()))
    kh2, vh2 = inc.dequantize(lens, int(lens.max()))
    np.testing.assert_array_equal(kh1, kh2)
    np.testing.assert_array_equal(vh1, vh2)


def test_ring_holds_between_w_and_w_plus_group_minus_one():
    """During single-token decode the bf16 residual grows from W to W+kg-1
    positions and drops back to W when a group is quantized: after every
    append, the positions from kg*floor((L-W)/kg) on come back exactly and
    the position before them (a quantized one) does not."""
    w = PC.with_(batch=1, window=8, k_group=16)
    total = 100
    kr, vr, kf, _, _, _ = wl.prefill(w, np.array([total], np.int32))
    c = _cache(w, [total])
    sizes = set()
    for L in range(total):
        c.append(kr[L:L + 1], vr[L:L + 1], oracle.IN_BF16, np.array([0, 1], np.int32), np.array([L], np.int32))
        Lnew = L + 1
        kh, _ = c.dequantize(np.array([Lnew], np.int32), Lnew)
        exact = np.all(kh[0, :, :Lnew] == kf[:Lnew].transpose(1, 0, 2), axis=(0, 2))
        Q = _paged(Lnew, 8, 16)
        assert exact[Q:].all()
        if Q:
            assert not exact[Q - 1]
            sizes.add(Lnew - Q)
    assert sizes == set(range(8, 24))


def test_outlier_channels_cost_less_with_position_groups():
    """With a few key channels ten times larger than the rest, per-token
    groups share the outlier's range with 31 other channels; groups along
    positions keep it to the outlier channel.  The key error of the ordinary
    channels is far lower with position groups."""
    w = PC.with_(batch=1, head_dim=128, window=0, k_bits=2, outliers=("random", 4, 10.0))
    L = 512
    kr, vr, kf, vf, cu, _ = wl.prefill(w, np.array([L], np.int32))
    out = {}
    for pc, G in ((False, 32), (True, 32)):
        wv = w.with_(k_per_channel=pc, k_group=G)
        c = _cache(wv, [L])
        c.append(kr, vr, oracle.IN_BF16, cu, np.zeros(1, np.int32))
        kh, _ = c.dequantize(np.array([L], np.int32), L)
        out[pc] = np.abs(kh[0, :, :L] - kf.transpose(1, 0, 2))
    ch = wl.outlier_channels(w)
    normal = np.ones((w.num_kv_heads, w.head_dim), bool)
    for h in range(w.num_kv_heads):
        normal[h, ch[h]] = False
    e_tok = out[False].transpose(0, 2, 1)[normal].mean()
    e_pc = out[True].transpose(0, 2, 1)[normal].mean()
    assert e_pc < 0.5 * e_tok


def test_attention_on_per_channel_cache():
    """Decode and chunked-prefill attention read the per-channel pages and
    the residual ring: library softmax over the dequantized rows."""
    w = PC.with_(window=16, k_group=32)
    lens = wl.lengths(w)
    c = _cache(w, lens)
    kr, vr, _, _, cu, _ = wl.prefill(w, lens)
    c.append(kr, vr, oracle.IN_BF16, cu, np.zeros(w.batch, np.int32))
    kh, vh = c.dequantize(lens, int(lens.max()))
    qr, qf = wl.query(w)
    sc = 1 / np.sqrt(w.head_dim)
    out, lse = c.decode_attention(qr, oracle.IN_BF16, lens, sc)
    n = np.minimum(lens, 20).astype(np.int32)
    cu_q = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    qc, qcf = wl.chunk_queries(w, int(cu_q[-1]))
    po, pl = c.prefill_attention(qc, oracle.IN_BF16, cu_q, lens, sc)
    g = w.gqa
    for b in range(w.batch):
        L = int(lens[b])
        for hq in range(w.num_q_heads):
            K = kh[b, hq // g, :L].astype(np.float64)
            V = vh[b, hq // g, :L].astype(np.float64)
            s = K @ qf[b, hq].astype(np.float64) * sc
            np.testing.assert_allclose(out[b, hq], scipy.special.softmax(s) @ V, rtol=1e-10, atol=1e-11)
            for i in range(int(n[b])):
                p = L - int(n[b]) + i
                row = int(cu_q[b]) + i
                s = K[:p + 1] @ qcf[row, hq].astype(np.float64) * sc
                np.testing.assert_allclose(po[row, hq], scipy.special.softmax(s) @ V[:p + 1], rtol=1e-10,
                                           atol=1e-11)


def test_unsupported_per_channel_layouts():
    with pytest.raises(ValueError):                       # groups must tile a page
        oracle.page_bytes(oracle.Layout(128, 8, 2, 4, 2, 48, 128, 64, 0, k_per_channel=True))
    with pytest.raises(ValueError):                       # rotation is a per-token channel mix
        oracle.page_bytes(oracle.Layout(128, 8, 2, 4, 2, 32, 128, 64, 0, rotate_keys=True,
                                        k_per_channel=True))


def test_storage_positions_hand_derived():
    """Per-channel key storage, derived by hand from the layout: key codes are
    channel runs of 64*kb/8 bytes stored like value runs (16-byte chunks,
    chunk-major), key metadata [64/kg][d] words.  K4 at head_dim 128: token
    slot 37 of channel 9 is the high nibble of run byte 18 = chunk 1, byte 2
    -> block offset 1*(128*16) + 9*16 + 2 = 2194.  With groups of 16
    positions, slot 37 is in group 2, so channel 9's metadata word is word
    2*128 + 9 = 265 of the block, bytes 1060..1063."""
    d = 128
    lay = oracle.Layout(d, 1, 1, 4, 4, 16, 128, 64, 0, k_per_channel=True)
    pt = np.zeros((1, 1), np.int32)
    c = oracle.Cache(lay, 1, pt, 1)
    # each channel's groups range over 0..15 (scale 1, zero 0): code == value
    k = np.zeros((64, 1, d), np.float32)
    v = np.zeros((64, 1, d), np.float32)
    k[15::16, 0, :] = 15.0                   # the last slot of every 16-position group
    k[37, 0, 9] = 6.0
    v[:, 0, 127] = 15.0
    c.append(k, v, oracle.IN_F32, np.array([0, 64], np.int32), np.zeros(1, np.int32))
    kb = c.k_codes.ravel()
    assert (kb[2194] >> 4) == 6
    assert (kb[2194] & 0x0F) == 0            # slot 36 of channel 9
    assert (kb[2194 + 16] >> 4) == 0         # slot 37 of channel 10
    meta = c.k_meta.view(np.uint8).ravel()
    scale = int(meta[1060]) | (int(meta[1061]) << 8)
    zero = int(meta[1062]) | (int(meta[1063]) << 8)
    assert (scale, zero) == (0x3C00, 0x0000)    # fp16 1.0 and +0
