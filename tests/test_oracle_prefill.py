"""Pins of the oracle's chunked-prefill attention (causal attention of a
chunk of new query tokens over the quantized cache).

"Kuantisasi KV cache mengganggu attention ...": section "Error pada key
masuk sebelum softmax" defines s = qK^T/sqrt(d), a = softmax(s), o = aV for
one new query; section "Pertumbuhan cache mengubah trade pada serving" says
the stored approximation is what later attention reads.  A chunk of n new
tokens is read as n such queries, query i seeing the positions up to its
own.  Each pin below checks that reading against something other than the
oracle's own attention loop: library softmax over exact or dequantized rows,
a closed form, or a perturbation that a wrong causal bound would expose.
"""
import numpy as np
import pytest
import scipy.linalg
import scipy.special

import oracle
import workloads as wl

SMALL = wl.Workload(name="small", batch=3, num_q_heads=6, num_kv_heads=2, head_dim=64,
                    seq_len=0, k_bits=4, v_bits=2, k_group=32, v_group=64, window=16,
                    ragged=(1, 200), shuffle_pages=True, outliers=("random", 2, 10.0), seed=3)


def _cache(w, lens, signs=None):
    pt = wl.page_table(w, lens)
    c = oracle.Cache(oracle.Layout.from_workload(w, signs), w.batch, pt, max(1, int((pt >= 0).sum())))
    return c


def _fill(w, lens, c, kr=None, vr=None):
    k0, v0, kf, vf, cu, _ = wl.prefill(w, lens)
    kr = k0 if kr is None else kr
    vr = v0 if vr is None else vr
    c.append(kr, vr, oracle.IN_BF16, cu, np.zeros(w.batch, np.int32))
    return kf, vf, cu


def _chunk(lens, cap):
    n = np.minimum(lens, cap).astype(np.int32)
    return n, np.concatenate([[0], np.cumsum(n)]).astype(np.int32)


def test_all_window_causal_chunk_is_exact_attention():
    """16-bit storage: every query of the chunk gets exact softmax attention
    over the bf16 rows up to its own position."""
    w = SMALL.with_(window=4096)
    lens = wl.lengths(w)
    c = _cache(w, lens)
    kf, vf, cu = _fill(w, lens, c)
    n, cu_q = _chunk(lens, 37)
    qr, qf = wl.chunk_queries(w, int(cu_q[-1]))
    sc = 1 / np.sqrt(w.head_dim)
    out, lse = c.prefill_attention(qr, oracle.IN_BF16, cu_q, lens, sc)
    g = w.gqa
    for b in range(w.batch):
        L = int(lens[b])
        for i in range(int(n[b])):
            p = L - int(n[b]) + i
            row = int(cu_q[b]) + i
            for hq in range(w.num_q_heads):
                K = kf[cu[b]:cu[b] + p + 1, hq // g].astype(np.float64)
                V = vf[cu[b]:cu[b] + p + 1, hq // g].astype(np.float64)
                s = K @ qf[row, hq].astype(np.float64) * sc
                np.testing.assert_allclose(out[row, hq], scipy.special.softmax(s) @ V, rtol=1e-11, atol=1e-12)
                assert abs(lse[row, hq] - scipy.special.logsumexp(s)) < 1e-10


@pytest.mark.parametrize("window,rotate", [(0, False), (16, False), (0, True), (16, True)])
def test_causal_chunk_on_reconstructed_cache(window, rotate):
    """Quantized and mixed caches: query i of a chunk equals library softmax
    over the dequantized rows [0, p]; with key rotation, page rows are scored
    with the rotated query and window rows with the plain one."""
    w = SMALL.with_(window=window, rotate_keys=rotate)
    lens = wl.lengths(w)
    signs = wl.rotation_signs(w) if rotate else None
    c = _cache(w, lens, signs)
    _fill(w, lens, c)
    kh, vh = c.dequantize(lens, int(lens.max()))
    n, cu_q = _chunk(lens, 70)                     # chunks longer than the window
    qr, qf = wl.chunk_queries(w, int(cu_q[-1]), step=1)
    sc = 1 / np.sqrt(w.head_dim)
    out, lse = c.prefill_attention(qr, oracle.IN_BF16, cu_q, lens, sc)
    H = scipy.linalg.hadamard(w.head_dim) / np.sqrt(w.head_dim)
    g = w.gqa
    for b in range(w.batch):
        L = int(lens[b])
        nq = max(0, L - window)
        for i in range(int(n[b])):
            p = L - int(n[b]) + i
            row = int(cu_q[b]) + i
            for hq in range(w.num_q_heads):
                q = qf[row, hq].astype(np.float64)
                K = kh[b, hq // g, :p + 1].astype(np.float64)
                V = vh[b, hq // g, :p + 1].astype(np.float64)
                s = K @ q
                if rotate:
                    m = min(nq, p + 1)
                    s[:m] = K[:m] @ ((q * signs) @ H)
                s *= sc
                np.testing.assert_allclose(out[row, hq], scipy.special.softmax(s) @ V, rtol=1e-10, atol=1e-11)
                assert abs(lse[row, hq] - scipy.special.logsumexp(s)) < 1e-9


def test_later_positions_do_not_reach_earlier_queries():
    """Changing only the newest token of each sequence leaves every other
    query of the chunk bit-identical and changes the newest query."""
    w = SMALL
    lens = wl.lengths(w)
    lens[0] = max(int(lens[0]), 40)
    k0, v0, _, _, cu, _ = wl.prefill(w, lens)
    k1, v1 = k0.copy(), v0.copy()
    r = np.random.default_rng(11)
    for b in range(w.batch):
        last = int(cu[b + 1]) - 1
        k1[last] = wl.bf16_bits(r.standard_normal(k1[last].shape, dtype=np.float32) * 3)
        v1[last] = wl.bf16_bits(r.standard_normal(v1[last].shape, dtype=np.float32) * 3)
    a, bb = _cache(w, lens), _cache(w, lens)
    _fill(w, lens, a)
    _fill(w, lens, bb, k1, v1)
    n, cu_q = _chunk(lens, 40)
    qr, _ = wl.chunk_queries(w, int(cu_q[-1]), step=2)
    sc = 1 / np.sqrt(w.head_dim)
    oa, la = a.prefill_attention(qr, oracle.IN_BF16, cu_q, lens, sc)
    ob, lb = bb.prefill_attention(qr, oracle.IN_BF16, cu_q, lens, sc)
    for b in range(w.batch):
        lo, hi = int(cu_q[b]), int(cu_q[b + 1])
        np.testing.assert_array_equal(oa[lo:hi - 1], ob[lo:hi - 1])
        np.testing.assert_array_equal(la[lo:hi - 1], lb[lo:hi - 1])
        assert not np.array_equal(oa[hi - 1], ob[hi - 1])


@pytest.mark.parametrize("window", [0, 16])
def test_newest_query_equals_decode_attention(window):
    """The last query of each chunk sees the whole sequence: it is the
    decode case."""
    w = SMALL.with_(window=window)
    lens = wl.lengths(w)
    c = _cache(w, lens)
    _fill(w, lens, c)
    n, cu_q = _chunk(lens, 9)
    qr, _ = wl.chunk_queries(w, int(cu_q[-1]), step=3)
    sc = 1 / np.sqrt(w.head_dim)
    out, lse = c.prefill_attention(qr, oracle.IN_BF16, cu_q, lens, sc)
    last = cu_q[1:] - 1
    od, ld = c.decode_attention(np.ascontiguousarray(qr[last]), oracle.IN_BF16, lens, sc)
    np.testing.assert_array_equal(out[last], od)
    np.testing.assert_array_equal(lse[last], ld)


def test_first_position_sees_only_itself():
    """A chunk that is the whole sequence: query 0 attends to position 0
    alone, so o = v_0 and lse = s_00 (closed form)."""
    w = SMALL.with_(window=0)
    lens = wl.lengths(w)
    c = _cache(w, lens)
    _fill(w, lens, c)
    kh, vh = c.dequantize(lens, int(lens.max()))
    n, cu_q = _chunk(lens, 10 ** 6)
    qr, qf = wl.chunk_queries(w, int(cu_q[-1]), step=4)
    sc = 1 / np.sqrt(w.head_dim)
    out, lse = c.prefill_attention(qr, oracle.IN_BF16, cu_q, lens, sc)
    for b in range(w.batch):
        row = int(cu_q[b])
        for hq in range(w.num_q_heads):
            h = hq // w.gqa
            np.testing.assert_array_equal(out[row, hq], vh[b, h, 0].astype(np.float64))
            s00 = float(kh[b, h, 0].astype(np.float64) @ qf[row, hq].astype(np.float64)) * sc
            assert abs(lse[row, hq] - s00) <= 1e-12 * max(1.0, abs(s00))


def test_empty_chunks_and_argument_errors():
    w = SMALL.with_(window=8)
    lens = np.array([30, 0, 5], np.int32)
    c = _cache(w, lens)
    _fill(w, lens, c)
    cu_q = np.array([0, 3, 3, 3], np.int32)            # sequences 1 and 2 send no query
    qr, _ = wl.chunk_queries(w, 3)
    out, lse = c.prefill_attention(qr, oracle.IN_BF16, cu_q, lens, 0.125)
    assert out.shape == (3, w.num_q_heads, w.head_dim) and np.all(np.isfinite(lse))
    with pytest.raises(ValueError):                     # more queries than positions
        c.prefill_attention(wl.chunk_queries(w, 9)[0], oracle.IN_BF16,
                            np.array([0, 3, 3, 9], np.int32), lens, 0.125)
    with pytest.raises(ValueError):                     # decreasing offsets
        c.prefill_attention(qr, oracle.IN_BF16, np.array([0, 3, 2, 3], np.int32), lens, 0.125)
