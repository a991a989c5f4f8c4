"""Memory-budget planner (CPU): byte accounting against the pinned memory
figures, and the choice against a brute-force search of its error table."""
import os

import pytest

from mixed_precision_quantized_kvq_b200 import planner

GOLD = os.path.join(os.path.dirname(__file__), "golden", "memory_k4v2_vs_k4v4.txt")


def _gold():
    out = {}
    for line in open(GOLD):
        line = line.strip()
        if line and not line.startswith("#") and "=" in line:
            k, v = line.split("=")
            out[k.strip()] = float(v)
    return out


def test_bytes_match_memory_golden():
    g = _gold()
    assert planner.bytes_per_token_head(4, 2, 32, 128) == g["token_head_bytes_k4v2_g32_g128_d128"]
    assert planner.bytes_per_token_head(4, 4, 32, 128) == g["token_head_bytes_k4v4_g32_g128_d128"]


def test_per_channel_bytes_match_golden():
    g = {}
    for line in open(os.path.join(os.path.dirname(GOLD), "memory_per_channel_keys.txt")):
        if "=" in line and not line.startswith("#"):
            k, v = line.split("=")
            g[k.strip()] = float(v)
    assert planner.bytes_per_token_head(4, 2, 64, 128, k_per_channel=True) == g["token_head_bytes_k4_pc64_v2_g128_d128"]
    assert planner.bytes_per_token_head(4, 2, 32, 128, k_per_channel=True) == g["token_head_bytes_k4_pc32_v2_g128_d128"]
    assert planner.bytes_per_token_head(2, 2, 64, 128, k_per_channel=True) == g["token_head_bytes_k2_pc64_v2_g128_d128"]


def test_table_has_both_key_grouping_axes():
    rows = planner.load_table()
    axes = {(r["k_bits"], r["v_bits"], bool(r.get("k_per_channel"))) for r in rows if r["k_group"] == 32}
    for kb in (1, 2, 4, 8):
        assert (kb, 1, False) in axes and (kb, 1, True) in axes


def test_table_covers_key_heavy_settings():
    rows = planner.load_table()
    keys = {(r["k_bits"], r["v_bits"], r["k_group"], r["v_group"]) for r in rows}
    for kb in (1, 2, 4, 8):
        for vb in (1, 2, 4, 8):
            if vb <= kb:
                assert (kb, vb, 32, 128) in keys
    assert all(r["v_bits"] <= r["k_bits"] for r in rows)


@pytest.mark.parametrize("budget", [60, 84, 100, 116, 148, 200, 300])
@pytest.mark.parametrize("metric", ["mean_abs", "max_abs"])
def test_plan_is_the_best_fitting_setting(budget, metric):
    rows = planner.load_table()
    fitting = [r for r in rows if r["v_bits"] <= r["k_bits"] and
               planner.bytes_per_token_head(r["k_bits"], r["v_bits"], r["k_group"], r["v_group"],
                                            k_per_channel=r.get("k_per_channel", False)) <= budget]
    if not fitting:
        with pytest.raises(ValueError):
            planner.plan(budget, metric)
        return
    best = min(r[metric] for r in fitting)
    p = planner.plan(budget, metric)
    assert p["bytes"] <= budget
    assert p[metric] == best
    assert p["k_bits"] >= p["v_bits"]


def test_frontier_is_monotone():
    f = planner.frontier()
    assert all(a["bytes"] <= b["bytes"] and a["mean_abs"] > b["mean_abs"] for a, b in zip(f, f[1:]))


def test_tiny_budget_is_refused():
    with pytest.raises(ValueError):
        planner.plan(1.0)
