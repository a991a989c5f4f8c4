"""Seeded synthetic inputs for the quantized KV-cache path.

This module is shared by the CPU oracle's tests, the CUDA path's tests, the
benchmark and the smoke check.  It only draws numbers and lays them out; it
holds none of the quantization or attention arithmetic.

Every array comes from ``numpy.random.default_rng([seed, stream, ...])`` with
a separate stream per quantity, so a subset (one sequence, one decode step)
can be regenerated on its own.  Floating-point draws are made in fp32 and,
where a workload says bf16, rounded to bf16 (round to nearest, ties to even)
as a data-preparation step; the bf16 bit patterns are what both sides read.

The five workloads follow the shapes the source pages work with: a
Llama-3-8B-like decode layer (32 query heads over 8 KV heads, head_dim 128),
a bit-allocation sweep at long context ("Quantize What Counts", results on
K4V2 vs K4V4 and 1-8 bit widths), a ragged paged serving batch with a recent
bf16 window ("kuantisasi KV cache ...", section on cache growth), and a
key-only Walsh-Hadamard rotation variant ("Quantize What Counts", rotation
integration).  Key outlier channels model the per-group outlier effect the
tag-index teasers describe.  No dataset item is reproduced: the public
benchmarks the pages name are replaced by these shapes.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field
from typing import Optional, Sequence

import numpy as np

# independent random streams
STREAM_K = 1
STREAM_OUTLIER = 2
STREAM_V = 3
STREAM_Q = 4
STREAM_LENS = 5
STREAM_PAGES = 6
STREAM_SIGNS = 7
STREAM_NEW_K = 8
STREAM_NEW_V = 9
STREAM_CHUNK_Q = 10

PAGE_SIZE = 64

DT_F32 = "f32"
DT_BF16 = "bf16"


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    seq_len: int                       # cached tokens per sequence (uniform case)
    k_bits: int = 4
    v_bits: int = 2
    k_group: int = 32
    v_group: int = 128
    window: int = 0
    page_size: int = PAGE_SIZE
    rotate_keys: bool = False
    k_per_channel: bool = False        # key groups of k_group positions of one channel
    in_dtype: str = DT_BF16
    # key outliers: ("fixed", (channels...), factor) | ("random", count, factor)
    #               | ("student_t", count, scale, nu)
    outliers: tuple = ("random", 4, 10.0)
    ragged: Optional[tuple] = None     # (lo, hi) inclusive uniform lengths
    shuffle_pages: bool = False
    decode_steps: int = 0
    seed: int = 0

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def gqa(self) -> int:
        return self.num_q_heads // self.num_kv_heads


TINY = Workload(
    name="tiny_k4v2_d64_l256", batch=1, num_q_heads=4, num_kv_heads=4,
    head_dim=64, seq_len=256, k_bits=4, v_bits=2, k_group=32, v_group=64,
    window=0, in_dtype=DT_F32, outliers=("fixed", (3, 17), 8.0))

LLAMA8B = Workload(
    name="llama3_8b_layer_b16_l4096_k4v2_w128", batch=16, num_q_heads=32,
    num_kv_heads=8, head_dim=128, seq_len=4096, k_bits=4, v_bits=2,
    k_group=32, v_group=128, window=128, outliers=("random", 4, 10.0))

SWEEP_BITS = ((8, 8), (4, 4), (4, 2), (2, 4), (2, 2), (1, 2))
SWEEP = Workload(
    name="sweep_b8_l16384", batch=8, num_q_heads=32, num_kv_heads=8,
    head_dim=128, seq_len=16384, k_group=32, v_group=128, window=0,
    outliers=("random", 4, 10.0))

RAGGED = Workload(
    name="ragged_paged_64seq_l512_16384_g5_w64", batch=64, num_q_heads=40,
    num_kv_heads=8, head_dim=128, seq_len=16384, ragged=(512, 16384),
    window=64, shuffle_pages=True, decode_steps=32,
    outliers=("random", 4, 10.0))

ROTATION = Workload(
    name="rotation_b32_l8192_k4v2", batch=32, num_q_heads=32, num_kv_heads=8,
    head_dim=128, seq_len=8192, window=0, rotate_keys=True,
    outliers=("student_t", 4, 10.0, 3.0))

ALL = {w.name: w for w in (TINY, LLAMA8B, SWEEP, RAGGED, ROTATION)}


def sweep_variants(base: Workload = SWEEP):
    return [base.with_(k_bits=kb, v_bits=vb, name=f"{base.name}_k{kb}v{vb}")
            for kb, vb in SWEEP_BITS]


# ---------------------------------------------------------------- helpers

def rng(seed: int, *stream: int) -> np.random.Generator:
    return np.random.default_rng([seed, *stream])


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest, ties to even (finite input)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    u = u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))
    return (u >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def lengths(w: Workload) -> np.ndarray:
    if w.ragged is None:
        return np.full(w.batch, w.seq_len, dtype=np.int32)
    lo, hi = w.ragged
    return rng(w.seed, STREAM_LENS).integers(lo, hi + 1, size=w.batch).astype(np.int32)


def outlier_channels(w: Workload) -> np.ndarray:
    """[num_kv_heads][count] channel indices of key outliers."""
    kind = w.outliers[0]
    if kind == "fixed":
        ch = np.asarray(w.outliers[1], dtype=np.int64)
        return np.tile(ch, (w.num_kv_heads, 1))
    count = int(w.outliers[1])
    g = rng(w.seed, STREAM_OUTLIER)
    return np.stack([g.choice(w.head_dim, size=count, replace=False)
                     for _ in range(w.num_kv_heads)]).astype(np.int64)


def _apply_outliers(w: Workload, k: np.ndarray, g: np.random.Generator) -> None:
    """k: [tokens][Hkv][d] fp32, modified in place."""
    ch = outlier_channels(w)
    kind = w.outliers[0]
    for h in range(w.num_kv_heads):
        if kind in ("fixed", "random"):
            k[:, h, ch[h]] *= np.float32(w.outliers[-1])
        elif kind == "student_t":
            scale, nu = w.outliers[2], w.outliers[3]
            t = g.standard_t(nu, size=(k.shape[0], ch.shape[1])).astype(np.float32)
            k[:, h, ch[h]] = np.float32(scale) * t
        else:
            raise ValueError(kind)


def _finish(w: Workload, x: np.ndarray):
    """Returns (array to hand to the library, fp32 values it represents)."""
    if w.in_dtype == DT_BF16:
        b = bf16_bits(x)
        return b, bf16_to_f32(b)
    x = np.ascontiguousarray(x, dtype=np.float32)
    return x, x


def seq_kv(w: Workload, b: int, n: int, start: int = 0):
    """Keys and values of positions [start, start+n) of sequence b.

    Returns (k_raw, v_raw, k_f32, v_f32), each [n][Hkv][d].  Draws are made
    for the whole prefix [0, start+n) so any window of positions is
    reproducible.
    """
    total = start + n
    gk = rng(w.seed, STREAM_K, b)
    k = gk.standard_normal((total, w.num_kv_heads, w.head_dim), dtype=np.float32)
    _apply_outliers(w, k, rng(w.seed, STREAM_OUTLIER, 1000 + b))
    gv = rng(w.seed, STREAM_V, b)
    v = gv.standard_normal((total, w.num_kv_heads, w.head_dim), dtype=np.float32)
    k, v = k[start:], v[start:]
    kr, kf = _finish(w, k)
    vr, vf = _finish(w, v)
    return kr, vr, kf, vf


def prefill(w: Workload, lens: Optional[np.ndarray] = None, with_f32: bool = True):
    """Ragged prefill batch: (k_raw, v_raw, k_f32, v_f32, cu_new, lens).

    k_raw is [sum(lens)][Hkv][d] (bf16 bits as uint16, or fp32); cu_new is the
    exclusive prefix sum [B+1].  With with_f32=False the fp32 views are None
    (saves host memory on the large workloads).
    """
    if lens is None:
        lens = lengths(w)
    lens = np.asarray(lens, dtype=np.int32)
    cu = np.zeros(w.batch + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lens)
    total = int(cu[-1])
    shape = (total, w.num_kv_heads, w.head_dim)
    rdt = np.uint16 if w.in_dtype == DT_BF16 else np.float32
    kr = np.empty(shape, rdt)
    vr = np.empty(shape, rdt)
    kf = np.empty(shape, np.float32) if with_f32 else None
    vf = np.empty(shape, np.float32) if with_f32 else None
    for b in range(w.batch):
        if lens[b] == 0:
            continue
        a, e = int(cu[b]), int(cu[b + 1])
        k_raw, v_raw, k_f, v_f = seq_kv(w, b, int(lens[b]))
        kr[a:e], vr[a:e] = k_raw, v_raw
        if with_f32:
            kf[a:e], vf[a:e] = k_f, v_f
    return kr, vr, kf, vf, cu, lens


def new_tokens(w: Workload, step: int):
    """One appended token per sequence for decode step `step`: [B][Hkv][d]."""
    k = rng(w.seed, STREAM_NEW_K, step).standard_normal(
        (w.batch, w.num_kv_heads, w.head_dim), dtype=np.float32)
    _apply_outliers(w, k, rng(w.seed, STREAM_OUTLIER, 2000 + step))
    v = rng(w.seed, STREAM_NEW_V, step).standard_normal(
        (w.batch, w.num_kv_heads, w.head_dim), dtype=np.float32)
    kr, kf = _finish(w, k)
    vr, vf = _finish(w, v)
    return kr, vr, kf, vf


def query(w: Workload, step: int = 0):
    """One query token per sequence: [B][Hq][d] (raw, f32)."""
    q = rng(w.seed, STREAM_Q, step).standard_normal(
        (w.batch, w.num_q_heads, w.head_dim), dtype=np.float32)
    return _finish(w, q)


def chunk_queries(w: Workload, total: int, step: int = 0):
    """Query rows of a chunk of new tokens, [total][Hq][d] (raw, f32)."""
    q = rng(w.seed, STREAM_CHUNK_Q, step).standard_normal(
        (total, w.num_q_heads, w.head_dim), dtype=np.float32)
    return _finish(w, q)


def rotation_signs(w: Workload) -> np.ndarray:
    """Seeded +-1 diagonal (int8, [head_dim]) shared by all heads of the layer."""
    g = rng(w.seed, STREAM_SIGNS)
    return np.where(g.integers(0, 2, size=w.head_dim) == 0, 1, -1).astype(np.int8)


def pages_needed(length: int, window: int, page_size: int = PAGE_SIZE) -> int:
    q = max(0, length - window)
    return (q + page_size - 1) // page_size


def page_table(w: Workload, capacity: Sequence[int]) -> np.ndarray:
    """[B][max_pages] physical page ids; sequence b gets ceil(capacity[b]/P)
    logical pages.  With shuffle_pages the physical ids are a seeded random
    permutation of all pages; unused entries are -1."""
    need = [(int(c) + w.page_size - 1) // w.page_size for c in capacity]
    maxp = max(1, max(need))
    total = int(sum(need))
    ids = np.arange(total, dtype=np.int32)
    if w.shuffle_pages:
        ids = rng(w.seed, STREAM_PAGES).permutation(total).astype(np.int32)
    pt = np.full((w.batch, maxp), -1, dtype=np.int32)
    o = 0
    for b, n in enumerate(need):
        pt[b, :n] = ids[o:o + n]
        o += n
    return pt


def check_fp16_metadata_range(x_f32: np.ndarray, bits: int) -> None:
    """Precondition of fp16 scale/zero storage: group minima >= -65504 and
    (max - min) / (2^bits - 1) <= 65504.  Checked over whole rows, which
    bounds every group inside them."""
    mn = float(x_f32.min()) if x_f32.size else 0.0
    mx = float(x_f32.max()) if x_f32.size else 0.0
    assert mn >= -65504.0, "input below fp16 range"
    assert (mx - mn) / (2 ** bits - 1) <= 65504.0, "group range too wide for fp16 scale"
