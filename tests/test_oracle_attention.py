"""Pins of the oracle's fp64 attention and its key-only rotation.

"Kuantisasi KV cache mengganggu attention ...", section "Error pada key masuk
sebelum softmax": s = qK^T/sqrt(d), a = softmax(s), o = aV, and a key error
E_K shifts the scores by qE_K^T/sqrt(d); section "Error pada value masuk
setelah bobot attention terbentuk": a value error E_V shifts the output by
aE_V with the weights unchanged.  Pins: scipy's softmax and numpy matmul as
an independent evaluation, closed forms (one token, zero query, a dominant
score, a constant score shift), and the two error identities.

"Quantize What Counts ..." (Resultaten, rotation on keys only): the
Sylvester Hadamard matrix is compared with scipy.linalg.hadamard and the
rotation with a numpy product; rotating both q and k preserves scores.
"""
import numpy as np
import scipy.linalg
import scipy.special

import oracle


def ref_attention(q, K, V, scale):
    s = (K @ q) * scale
    a = scipy.special.softmax(s)
    return a @ V, scipy.special.logsumexp(s), a, s


def test_matches_scipy():
    r = np.random.default_rng(1)
    for L, d in ((1, 64), (7, 64), (300, 128), (1000, 128)):
        q = r.standard_normal(d)
        K = r.standard_normal((L, d)) * 3
        V = r.standard_normal((L, d))
        o, lse = oracle.attention_dense(q, K, V, 1 / np.sqrt(d))
        o_ref, lse_ref, _, _ = ref_attention(q, K, V, 1 / np.sqrt(d))
        np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-13)
        assert abs(lse - lse_ref) < 1e-11


def test_closed_forms():
    r = np.random.default_rng(2)
    d = 64
    v = r.standard_normal((1, d))
    k = r.standard_normal((1, d))
    q = r.standard_normal(d)
    o, lse = oracle.attention_dense(q, k, v, 0.125)
    np.testing.assert_array_equal(o, v[0])                       # one token: o = v
    assert abs(lse - 0.125 * float(k[0] @ q)) < 1e-12             # lse = its score
    K = r.standard_normal((50, d))
    V = r.standard_normal((50, d))
    o, lse = oracle.attention_dense(np.zeros(d), K, V, 0.125)
    np.testing.assert_allclose(o, V.mean(0), rtol=1e-12, atol=1e-14)  # uniform weights
    assert abs(lse - np.log(50)) < 1e-12
    K2 = K.copy()
    K2[17] = q * 100                                              # one dominant score
    o, _ = oracle.attention_dense(q, K2, V, 1.0)
    np.testing.assert_allclose(o, V[17], rtol=0, atol=1e-12)
    # a constant shift of every score leaves o unchanged and moves lse
    qe = np.concatenate([q, [1.0]])
    Ke = np.concatenate([K, np.full((50, 1), 7.0)], axis=1)
    o1, l1 = oracle.attention_dense(q, K, V, 0.5)
    Ve = np.concatenate([V, np.zeros((50, 1))], axis=1)
    o2, l2 = oracle.attention_dense(qe, Ke, Ve, 0.5)
    np.testing.assert_allclose(o1, o2[:d], rtol=1e-12, atol=1e-14)
    assert abs((l2 - l1) - 3.5) < 1e-11
    o, lse = oracle.attention_dense(q, np.zeros((0, d)), np.zeros((0, d)), 1.0)
    assert np.all(o == 0) and lse == -np.inf                     # empty sequence


def _scores(q, K, scale):
    return np.array([oracle.attention_dense(q, K[t:t + 1], np.zeros((1, len(q))), scale)[1]
                     for t in range(K.shape[0])])


def test_key_error_enters_before_softmax():
    r = np.random.default_rng(3)
    d, L = 128, 40
    q, K, V = r.standard_normal(d), r.standard_normal((L, d)), r.standard_normal((L, d))
    EK = r.standard_normal((L, d)) * 0.05
    sc = 1 / np.sqrt(d)
    s, s2 = _scores(q, K, sc), _scores(q, K + EK, sc)
    np.testing.assert_allclose(s2 - s, (EK @ q) * sc, rtol=1e-9, atol=1e-12)
    # and the output changes through the weights, not linearly in E_K
    o, _ = oracle.attention_dense(q, K, V, sc)
    o2, _ = oracle.attention_dense(q, K + EK, V, sc)
    a2 = scipy.special.softmax(s2)
    np.testing.assert_allclose(o2, a2 @ V, rtol=1e-11, atol=1e-13)


def test_value_error_enters_after_weights():
    r = np.random.default_rng(4)
    d, L = 128, 40
    q, K, V = r.standard_normal(d), r.standard_normal((L, d)), r.standard_normal((L, d))
    EV = r.standard_normal((L, d)) * 0.05
    sc = 1 / np.sqrt(d)
    o, lse = oracle.attention_dense(q, K, V, sc)
    o2, lse2 = oracle.attention_dense(q, K, V + EV, sc)
    a = scipy.special.softmax((K @ q) * sc)
    np.testing.assert_allclose(o2 - o, a @ EV, rtol=1e-9, atol=1e-13)
    assert lse == lse2                                            # weights unchanged


def test_hadamard_matches_scipy_sylvester():
    for n in (64, 128):
        H = oracle.hadamard(n)
        np.testing.assert_array_equal(H, scipy.linalg.hadamard(n).astype(np.float64))
        np.testing.assert_array_equal(H @ H.T, n * np.eye(n))


def test_rotation_matches_numpy_and_preserves_scores():
    r = np.random.default_rng(6)
    d = 128
    signs = np.where(r.integers(0, 2, d) == 0, 1, -1).astype(np.int8)
    x = (r.standard_normal((20, d)) * 5).astype(np.float32)
    y = oracle.rotate(x, signs)
    want = (x.astype(np.float64) * signs) @ scipy.linalg.hadamard(d) / np.sqrt(d)
    np.testing.assert_array_equal(y, want.astype(np.float32))     # one rounding to fp32
    q = r.standard_normal(d)
    K = r.standard_normal((20, d))
    qr = (q * signs) @ scipy.linalg.hadamard(d) / np.sqrt(d)
    Kr = (K * signs) @ scipy.linalg.hadamard(d) / np.sqrt(d)
    np.testing.assert_allclose(Kr @ qr, K @ q, rtol=1e-12, atol=1e-12)
