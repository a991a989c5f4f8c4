"""Quantization-induced attention error on synthetic KV caches.

TEST INFRASTRUCTURE ONLY (like the rest of ``oracle/``): it uses the oracle's
group quantizer and fp64 numpy attention, never the CUDA library.

This is a report, not a parity check.  It measures how far attention over
the quantized cache moves from attention over the exact bf16 cache, for one
sequence of a workload, as the two pages describe it:
  * "Kuantisasi KV cache mengganggu attention melalui key dan value
    tersimpan", sections "Error pada key masuk sebelum softmax" (key error
    shifts the scores, s' = s + q E_K^T / sqrt(d), and so the weights) and
    "Error pada value masuk setelah bobot attention terbentuk" (value error
    is averaged by the weights, o' = o + a E_V);
  * "Quantize What Counts: More for Keys, Less for Values", Resultaten
    (more bits for keys than values; rotation helps keys, not values).
Metrics per setting: max and mean |o' - o|, max |s' - s| over scores scaled
by 1/sqrt(d), the largest total-variation distance between a' and a over the
query heads, and the same output error with only the keys (key-only) or only
the values (value-only) quantized.

    python -m oracle.error_report            # markdown table on stdout
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np

if __package__ in (None, ""):
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import oracle  # noqa: E402
import workloads as wl  # noqa: E402


def _rotation_matrix(signs: np.ndarray) -> np.ndarray:
    """diag(signs) H / sqrt(d) in fp64 (orthogonal)."""
    d = signs.shape[0]
    return np.diag(signs.astype(np.float64)) @ oracle.hadamard(d) / np.sqrt(d)


def _quantized_rows(x: np.ndarray, group: int, bits: int) -> np.ndarray:
    """Rows of x through the oracle's group quantizer and back (fp64)."""
    s, z, c = oracle.quantize_rows(x.astype(np.float32), group, bits)
    return oracle.dequantize_rows(c, s, z, group).astype(np.float64)


def _quantized_columns(x: np.ndarray, group: int, bits: int) -> np.ndarray:
    """Columns of x [L][d] through the oracle's group quantizer in groups of
    `group` consecutive rows (positions) of one column (channel), and back."""
    L, d = x.shape
    assert L % group == 0
    return _quantized_rows(np.ascontiguousarray(x.T), group, bits).T


def _attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, g: int, scale: float):
    """q [Hq][d], K and V [L][Hkv][d] -> scores s [Hq][L], weights a, output o [Hq][d] (fp64)."""
    Hq = q.shape[0]
    kv = np.arange(Hq) // g
    s = np.einsum("hd,lhd->hl", q, K[:, kv, :]) * scale
    a = np.exp(s - s.max(axis=1, keepdims=True))
    a /= a.sum(axis=1, keepdims=True)
    o = np.einsum("hl,lhd->hd", a, V[:, kv, :])
    return s, a, o


def reconstruct(K: np.ndarray, V: np.ndarray, k_group: int, k_bits: int, v_group: int, v_bits: int,
                Rk: np.ndarray | None = None, Rv: np.ndarray | None = None, k_per_channel: bool = False):
    """Keys and values [L][Hkv][d] (fp64) as the quantized cache holds them,
    in the original basis.  Rk / Rv: an orthogonal rotation applied to the
    rows before quantization ("Quantize What Counts", Resultaten: rotation of
    keys, and as an ablation of values); the quantized rows x^ R^T map back,
    since R R^T = I.  k_per_channel: key groups of k_group positions of one
    channel."""
    L, Hkv, d = K.shape
    if Rk is not None:
        Kr = (K.reshape(-1, d) @ Rk).astype(np.float32)
        Khat = (_quantized_rows(Kr, k_group, k_bits) @ Rk.T).reshape(L, Hkv, d)
    elif k_per_channel:
        Khat = np.stack([_quantized_columns(K[:, h].astype(np.float32), k_group, k_bits)
                         for h in range(Hkv)], axis=1)
    else:
        Khat = _quantized_rows(K.reshape(-1, d), k_group, k_bits).reshape(L, Hkv, d)
    if Rv is not None:
        Vr = (V.reshape(-1, d) @ Rv).astype(np.float32)
        Vhat = _quantized_rows(Vr, v_group, v_bits) @ Rv.T
    else:
        Vhat = _quantized_rows(V.reshape(-1, d), v_group, v_bits)
    return Khat, Vhat.reshape(L, Hkv, d)


def measure(w: wl.Workload, k_bits: int, v_bits: int, rotate_keys: bool = False,
            rotate_values: bool = False, length: int | None = None, k_per_channel: bool = False) -> dict:
    """Error of attention over the quantized cache for one sequence of `w`.
    k_per_channel: key groups of w.k_group positions of one channel (the
    sequence length must be a multiple of it) instead of w.k_group channels
    of one token."""
    w1 = w.with_(batch=1, window=0, seq_len=length or w.seq_len or w.ragged[1], ragged=None,
                 rotate_keys=False, k_bits=k_bits, v_bits=v_bits)
    lens = wl.lengths(w1)
    _, _, kf, vf, _, _ = wl.prefill(w1, lens)
    L, d, Hkv = int(lens[0]), w1.head_dim, w1.num_kv_heads
    K = kf.reshape(L, Hkv, d).astype(np.float64)
    V = vf.reshape(L, Hkv, d).astype(np.float64)
    _, qf = wl.query(w1)
    q = qf[0].astype(np.float64)
    scale = 1.0 / np.sqrt(d)
    g = w1.num_q_heads // Hkv
    R = _rotation_matrix(wl.rotation_signs(w.with_(rotate_keys=True))) if (rotate_keys or rotate_values) else None
    Khat, Vhat = reconstruct(K, V, w1.k_group, k_bits, w1.v_group, v_bits, R if rotate_keys else None,
                             R if rotate_values else None, k_per_channel)

    s0, a0, o0 = _attention(q, K, V, g, scale)
    s1, a1, o1 = _attention(q, Khat, Vhat, g, scale)
    _, _, ok = _attention(q, Khat, V, g, scale)
    _, _, ov = _attention(q, K, Vhat, g, scale)
    err = np.abs(o1 - o0)
    return {
        "k_bits": k_bits, "v_bits": v_bits, "rotate_keys": rotate_keys, "rotate_values": rotate_values,
        "k_per_channel": k_per_channel, "k_group": w1.k_group,
        "tokens": L, "max_abs": float(err.max()), "mean_abs": float(err.mean()),
        "score_max_abs": float(np.abs(s1 - s0).max()),
        "tv_max": float(0.5 * np.abs(a1 - a0).sum(axis=1).max()),
        "key_only_max_abs": float(np.abs(ok - o0).max()),
        "value_only_max_abs": float(np.abs(ov - o0).max()),
        "o_abs_mean": float(np.abs(o0).mean()),
    }


def table(rows) -> str:
    head = ("| keys | values | rotation | max \\|o'-o\\| | mean \\|o'-o\\| | max \\|s'-s\\| | max TV(a', a) "
            "| key-only max | value-only max |\n|---|---|---|---:|---:|---:|---:|---:|---:|")
    out = [head]
    for r in rows:
        rot = "+".join(n for n, f in (("keys", r["rotate_keys"]), ("values", r["rotate_values"])) if f) or "none"
        kb = f"{r['k_bits']} ({r['k_group']} positions)" if r.get("k_per_channel") else f"{r['k_bits']}"
        out.append(f"| {kb} | {r['v_bits']} | {rot} | {r['max_abs']:.4f} | {r['mean_abs']:.5f} | "
                   f"{r['score_max_abs']:.4f} | {r['tv_max']:.4f} | {r['key_only_max_abs']:.4f} | "
                   f"{r['value_only_max_abs']:.4f} |")
    return "\n".join(out)


def grid(length: int = 4096):
    """Errors of every (key bits >= value bits, key grouping, value group)
    setting at head_dim 128 on the sweep workload's distribution: the table
    the memory-budget planner reads.  Key groupings: 32, 64 or 128 channels
    of one token, or 32 or 64 positions of one channel."""
    out = []
    for kb in (8, 4, 2, 1):
        for vb in (8, 4, 2, 1):
            if vb > kb:
                continue
            for pc, kgs in ((False, (32, 64, 128)), (True, (32, 64))):
                for kg in kgs:
                    for vg in (64, 128):
                        r = measure(wl.SWEEP.with_(k_group=kg, v_group=vg), kb, vb, length=length,
                                    k_per_channel=pc)
                        r.update(k_group=kg, v_group=vg)
                        out.append(r)
    return out


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--length", type=int, default=16384, help="tokens of the sequence")
    ap.add_argument("--grid-json", help="write the planner's error table (JSON) to this path and exit")
    args = ap.parse_args(argv)
    if args.grid_json:
        import json
        rows = grid(min(args.length, 4096))
        keep = ("k_bits", "v_bits", "k_group", "v_group", "k_per_channel", "tokens", "max_abs", "mean_abs",
                "score_max_abs", "tv_max")
        with open(args.grid_json, "w") as f:
            json.dump({"source": "python -m oracle.error_report --grid-json (oracle quantizer, fp64 attention, "
                                 "sweep workload distribution, one sequence, head_dim 128, 32/8 heads)",
                       "rows": [{k: r[k] for k in keep} for r in rows]}, f, indent=1)
        return
    rows = [measure(wl.SWEEP, kb, vb, length=args.length) for kb, vb in wl.SWEEP_BITS]
    print(f"sweep workload, one sequence of {args.length} tokens, 32/8 heads, d128, key groups 32, "
          "value groups 128; outlier key channels x10\n")
    print(table(rows))
    rot = [measure(wl.ROTATION, 4, 2, length=args.length, rotate_keys=rk, rotate_values=rv)
           for rk, rv in ((False, False), (True, False), (False, True), (True, True))]
    print(f"\nrotation workload (outlier key channels 10 * t(3)), K4V2, one sequence of {args.length} tokens\n")
    print(table(rot))
    pc = [measure(wl.SWEEP.with_(k_group=g), kb, 2, length=args.length, k_per_channel=per)
          for kb in (4, 2) for per, g in ((False, 32), (True, 32), (True, 64))]
    print(f"\nsweep workload, key groups of 32 channels of one token vs groups of 32 / 64 positions of one "
          f"channel, values 2-bit in groups of 128, one sequence of {args.length} tokens\n")
    print(table(pc))


if __name__ == "__main__":
    main()
