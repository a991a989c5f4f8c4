"""The quantization-error report (oracle side, CPU): sanity of its metrics on a
short sequence.  These are properties any correct report has, not the
pages' accuracy numbers (those need real models and stay unpinned)."""
import numpy as np
import pytest

from oracle import error_report as er
import workloads as wl


@pytest.fixture(scope="module")
def rows():
    return {(kb, vb): er.measure(wl.SWEEP, kb, vb, length=512) for kb, vb in
            [(8, 8), (4, 4), (4, 2), (2, 4), (2, 2)]}


def test_metrics_are_in_range(rows):
    for r in rows.values():
        assert 0.0 <= r["mean_abs"] <= r["max_abs"]
        assert 0.0 <= r["tv_max"] <= 1.0
        assert r["score_max_abs"] >= 0.0


def test_error_shrinks_with_bits(rows):
    assert rows[(8, 8)]["max_abs"] < rows[(4, 4)]["max_abs"] < rows[(2, 2)]["max_abs"]
    assert rows[(8, 8)]["mean_abs"] < rows[(4, 4)]["mean_abs"] < rows[(2, 2)]["mean_abs"]


def test_key_error_depends_on_key_bits_only(rows):
    """Scores and weights see only the keys ("Error pada key masuk sebelum
    softmax"): settings with the same key bits give the same score error and
    the same key-only output error; the value-only error follows the value bits."""
    assert rows[(4, 4)]["score_max_abs"] == rows[(4, 2)]["score_max_abs"]
    assert rows[(4, 4)]["key_only_max_abs"] == rows[(4, 2)]["key_only_max_abs"]
    assert rows[(2, 4)]["value_only_max_abs"] == rows[(4, 4)]["value_only_max_abs"]


def test_lossless_limit():
    """With 8-bit codes on a constant-free cache the output error is small
    against the output scale."""
    r = er.measure(wl.SWEEP, 8, 8, length=256)
    assert r["max_abs"] < 0.05 * max(1.0, r["o_abs_mean"] * 10)
    assert np.isfinite(r["tv_max"])


def test_per_channel_report_matches_the_cache():
    """The report's key groups along positions are the oracle cache's
    per-channel groups (window 0, length a multiple of the group)."""
    import numpy as np

    import oracle
    import workloads as wl
    from oracle import error_report as er

    w = wl.SWEEP.with_(batch=1, num_kv_heads=2, num_q_heads=8, window=0, k_group=32, k_per_channel=True)
    L = 256
    lens = np.array([L], np.int32)
    kr, vr, kf, _, cu, _ = wl.prefill(w, lens)
    pt = wl.page_table(w, lens)
    c = oracle.Cache(oracle.Layout.from_workload(w), 1, pt, int((pt >= 0).sum()))
    c.append(kr, vr, oracle.IN_BF16, cu, np.zeros(1, np.int32))
    kh, _ = c.dequantize(lens, L)
    for h in range(w.num_kv_heads):
        np.testing.assert_array_equal(er._quantized_columns(kf[:, h], 32, w.k_bits), kh[0, h])


# ---------------------------------------------------------------- rotation pins
# The report's rotation ("Quantize What Counts", Resultaten: keys rotated
# before quantization; values only as an ablation) must be the cache's
# rotation and must map back to the original basis.

def _signs():
    return wl.rotation_signs(wl.ROTATION)


def test_rotation_matrix_is_orthogonal():
    R = er._rotation_matrix(_signs())
    np.testing.assert_allclose(R @ R.T, np.eye(R.shape[0]), rtol=0, atol=1e-12)


def test_rotation_matrix_is_the_oracle_key_rotation():
    """Row i of diag(signs) H / sqrt(d) is the oracle's rotation of unit
    vector e_i (the C rotation pinned against scipy's Hadamard in
    test_oracle_attention), so the report rotates exactly like the cache:
    signs first, then H."""
    import oracle
    signs = _signs()
    d = signs.shape[0]
    R = er._rotation_matrix(signs)
    rot = oracle.rotate(np.eye(d, dtype=np.float32), signs)
    np.testing.assert_array_equal(rot, R.astype(np.float32))
    # and not the other order (H then signs), which is a different matrix
    Hd = oracle.hadamard(d) @ np.diag(signs.astype(np.float64)) / np.sqrt(d)
    assert np.abs(Hd.astype(np.float32) - rot).max() > 0.1


def _row_bound(X, Rk, group, bits):
    """Per-row 2-norm bound on |x^ R^T - x| from the quantizer's element
    bound |x_r - x^_r| <= scale/2 in the rotated basis (R orthogonal), plus
    fp32 rounding of the rotated rows and of the reconstruction."""
    import oracle
    Xr = (X @ Rk).astype(np.float32)
    s, _, _ = oracle.quantize_rows(Xr, group, bits)
    s = np.asarray(s, np.uint16).view(np.float16).astype(np.float64)   # binary16 scale bits
    per_el = np.repeat(s, group, axis=1) / 2 + 2 * np.spacing(np.abs(Xr).astype(np.float32)).astype(np.float64)
    return np.sqrt((per_el ** 2).sum(axis=1)) + 2 ** -22 * np.linalg.norm(X, axis=1)


@pytest.mark.parametrize("rot_keys,rot_values", [(True, False), (False, True), (True, True)])
def test_rotated_reconstruction_within_quantizer_bound(rot_keys, rot_values):
    """At 8 bits, keys and values rotated before quantization come back in the
    original basis within the quantizer's bound: a reconstruction with R in
    place of R^T, or a rotation applied to one side only, fails this."""
    w = wl.ROTATION.with_(batch=1, window=0, seq_len=192, rotate_keys=False)
    lens = wl.lengths(w)
    _, _, kf, vf, _, _ = wl.prefill(w, lens)
    L, d, Hkv = int(lens[0]), w.head_dim, w.num_kv_heads
    K = kf.reshape(L, Hkv, d).astype(np.float64)
    V = vf.reshape(L, Hkv, d).astype(np.float64)
    R = er._rotation_matrix(_signs())
    Khat, Vhat = er.reconstruct(K, V, w.k_group, 8, w.v_group, 8, R if rot_keys else None,
                                R if rot_values else None)
    for X, Xh, on, grp in ((K, Khat, rot_keys, w.k_group), (V, Vhat, rot_values, w.v_group)):
        X2, Xh2 = X.reshape(-1, d), Xh.reshape(-1, d)
        err = np.linalg.norm(Xh2 - X2, axis=1)
        bound = _row_bound(X2, R if on else np.eye(d), grp, 8)
        assert np.all(err <= bound), float((err / bound).max())
        # the bound is not vacuous: it is far below the rows' own size
        assert np.all(bound < 0.05 * np.linalg.norm(X2, axis=1) + 1e-3)


def test_rotated_measure_rows_are_consistent():
    """measure() with rotation runs through reconstruct(): key rotation
    changes only the key-side metrics, value rotation only the value-only
    error."""
    base = er.measure(wl.ROTATION, 4, 2, length=256)
    rk = er.measure(wl.ROTATION, 4, 2, rotate_keys=True, length=256)
    rv = er.measure(wl.ROTATION, 4, 2, rotate_values=True, length=256)
    assert rk["value_only_max_abs"] == base["value_only_max_abs"]
    assert rv["score_max_abs"] == base["score_max_abs"]
    assert rv["key_only_max_abs"] == base["key_only_max_abs"]
    assert rk["score_max_abs"] != base["score_max_abs"]
    assert rv["value_only_max_abs"] != base["value_only_max_abs"]
