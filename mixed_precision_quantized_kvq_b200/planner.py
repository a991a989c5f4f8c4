"""Memory-budget planner for the quantized KV cache.

"Quantize What Counts: More for Keys, Less for Values" (Belangrijkste
Bijdragen, Resultaten) argues that bits belong to the keys first: at a fixed
memory budget a key-heavy split (K4V2) beats an even one.  This module turns
that rule into a choice.  Given a budget in bytes per token and kv-head, it
picks the setting (key bits, value bits, key grouping, value group), with
key bits >= value bits, that fits the budget and has the smallest measured
attention error.  Key groups run either over channels of one token or over
positions of one channel ("Kuantisasi KV cache ...", section "Granularitas
kuantisasi menentukan nilai yang berbagi scale": the grouping axis is an
implementation choice).

* Bytes come from the library's own accounting (`kvq_page_bytes`: packed
  codes plus fp16 scale and zero point per group, "Kuantisasi KV cache ...",
  section "Pertumbuhan cache mengubah trade pada serving": memory is payload
  plus metadata).
* Errors come from `data/error_table.json`. That table is measured on
  synthetic caches of the benchmark workloads' shape (head_dim 128, 32/8
  heads, outlier key channels). It was written by the CPU reference's error
  report (`python -m oracle.error_report --grid-json ...`) and is shipped as
  plain data. The planner executes nothing of that reference.

    python -m mixed_precision_quantized_kvq_b200.planner --budget 116
"""
from __future__ import annotations

import argparse
import json
import os
from typing import Dict, List, Optional

from . import PAGE_SIZE, Layout, kvq_page_bytes

TABLE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "data", "error_table.json")
METRICS = ("mean_abs", "max_abs", "score_max_abs", "tv_max")


def bytes_per_token_head(k_bits: int, v_bits: int, k_group: int, v_group: int, head_dim: int = 128,
                         k_per_channel: bool = False) -> float:
    """Cache bytes of one token of one kv-head: codes and metadata of keys and
    values (k_per_channel: key groups of k_group positions of one channel)."""
    lay = Layout(head_dim, 1, 1, k_bits, v_bits, k_group, v_group, PAGE_SIZE, 0, k_per_channel=k_per_channel)
    kc, km, vc, vm = kvq_page_bytes(lay)
    return (kc + km + vc + vm) / PAGE_SIZE


def load_table(path: str = TABLE) -> List[Dict]:
    with open(path) as f:
        return json.load(f)["rows"]


def frontier(table: Optional[List[Dict]] = None, metric: str = "mean_abs", head_dim: int = 128) -> List[Dict]:
    """Every setting of the table with its bytes, sorted by bytes, keeping only
    those that lower the error below every cheaper setting (the Pareto front)."""
    rows = []
    for r in (table if table is not None else load_table()):
        if r["v_bits"] > r["k_bits"]:
            continue
        pc = bool(r.get("k_per_channel", False))
        b = bytes_per_token_head(r["k_bits"], r["v_bits"], r["k_group"], r["v_group"], head_dim, pc)
        rows.append(dict(r, bytes=b, k_per_channel=pc))
    rows.sort(key=lambda r: (r["bytes"], r[metric]))
    out, best = [], float("inf")
    for r in rows:
        if r[metric] < best:
            out.append(r)
            best = r[metric]
    return out


def plan(budget_bytes: float, metric: str = "mean_abs", table: Optional[List[Dict]] = None,
         head_dim: int = 128) -> Dict:
    """The setting with the smallest `metric` among those whose bytes per
    token and kv-head fit `budget_bytes` (ties: fewer bytes)."""
    if metric not in METRICS:
        raise ValueError(f"metric must be one of {METRICS}")
    fits = [r for r in frontier(table, metric, head_dim) if r["bytes"] <= budget_bytes]
    if not fits:
        raise ValueError(f"no setting fits {budget_bytes} bytes per token and kv-head")
    return min(fits, key=lambda r: (r[metric], r["bytes"]))


def main(argv=None):
    ap = argparse.ArgumentParser(description="choose key/value bits and groups for a memory budget")
    ap.add_argument("--budget", type=float, required=True, help="bytes per token and kv-head (head_dim 128)")
    ap.add_argument("--metric", default="mean_abs", choices=METRICS)
    args = ap.parse_args(argv)
    r = plan(args.budget, args.metric)
    print(f"{describe(r)}: {r['bytes']:.1f} B per token-head, {args.metric} {r[args.metric]:.5f}")
    print("\nfrontier (bytes -> error):")
    for f in frontier(metric=args.metric):
        print(f"  {f['bytes']:6.1f} B  {describe(f)}  {args.metric} {f[args.metric]:.5f}")


def describe(r: Dict) -> str:
    kgrp = f"{r['k_group']} positions" if r.get("k_per_channel") else f"g{r['k_group']}"
    return f"K{r['k_bits']} {kgrp} / V{r['v_bits']} g{r['v_group']}"


if __name__ == "__main__":
    main()
