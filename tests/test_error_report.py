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
