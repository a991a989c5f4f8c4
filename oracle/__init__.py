"""ctypes front end of the CPU oracle (``kvq_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by the test suite, the smoke check and
the benchmark's CPU-baseline leg.  The CUDA library and its Python binding
never import this package, and this package imports nothing from them.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from dataclasses import dataclass
from typing import Optional

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "kvq_oracle.c")
# KVQO_SANITIZE=1 builds and loads a separate copy under AddressSanitizer and
# UBSan (the process must preload libasan); the arithmetic flags are the same.
SANITIZE = os.environ.get("KVQO_SANITIZE") == "1"
LIB = os.path.join(HERE, "libkvq_oracle_sanitized.so" if SANITIZE else "libkvq_oracle.so")

RN, RD, RU = 0, -1, 1
IN_F32, IN_BF16 = 0, 1

CFLAGS = ["-O2", "-fPIC", "-shared", "-frounding-math", "-ffp-contract=off",
          "-fno-fast-math", "-fopenmp", "-Wall"]
if SANITIZE:
    CFLAGS += ["-g", "-fsanitize=address,undefined", "-fno-sanitize-recover=all", "-fno-omit-frame-pointer"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain C, no fast-math, no contraction)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + ".tmp"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, SRC, "-lm"])
        os.replace(tmp, LIB)
    return LIB


class _Layout(C.Structure):
    _fields_ = [("head_dim", C.c_int), ("num_q_heads", C.c_int), ("num_kv_heads", C.c_int),
                ("k_bits", C.c_int), ("v_bits", C.c_int), ("k_group", C.c_int),
                ("v_group", C.c_int), ("page_size", C.c_int), ("window", C.c_int),
                ("rotate_keys", C.c_int), ("rot_signs", C.c_void_p), ("k_per_channel", C.c_int)]


class _Cache(C.Structure):
    _fields_ = [("k_codes", C.c_void_p), ("v_codes", C.c_void_p), ("k_meta", C.c_void_p),
                ("v_meta", C.c_void_p), ("k_win", C.c_void_p), ("v_win", C.c_void_p),
                ("page_table", C.c_void_p), ("batch", C.c_int),
                ("max_pages_per_seq", C.c_int)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(LIB)
        P = C.c_void_p
        L.kvqo_f32_to_f16.restype = C.c_uint16
        L.kvqo_f32_to_f16.argtypes = [C.c_float, C.c_int]
        L.kvqo_f16_to_f32.restype = C.c_float
        L.kvqo_f16_to_f32.argtypes = [C.c_uint16]
        L.kvqo_f32_to_bf16.restype = C.c_uint16
        L.kvqo_f32_to_bf16.argtypes = [C.c_float, C.c_int]
        for n in ("kvqo_sub_ru", "kvqo_div_ru", "kvqo_sub_rn", "kvqo_div_rn"):
            getattr(L, n).restype = C.c_float
            getattr(L, n).argtypes = [C.c_float, C.c_float]
        L.kvqo_f32_to_f16_n.argtypes = [P, C.c_long, C.c_int, P]
        L.kvqo_f32_to_bf16_n.argtypes = [P, C.c_long, C.c_int, P]
        L.kvqo_op_n.argtypes = [P, P, C.c_long, C.c_int, C.c_int, P]
        L.kvqo_quantize_group.argtypes = [P, C.c_int, C.c_int, P, P, P]
        L.kvqo_quantize_rows.argtypes = [P, C.c_long, C.c_int, C.c_int, C.c_int, P, P, P]
        L.kvqo_dequantize_rows.argtypes = [P, P, P, C.c_long, C.c_int, C.c_int, P]
        L.kvqo_dequant_code.restype = C.c_float
        L.kvqo_dequant_code.argtypes = [C.c_uint8, C.c_uint16, C.c_uint16]
        L.kvqo_pack.argtypes = [P, C.c_int, C.c_int, P]
        L.kvqo_unpack_one.restype = C.c_uint8
        L.kvqo_unpack_one.argtypes = [P, C.c_int, C.c_int]
        L.kvqo_hadamard.argtypes = [C.c_int, P]
        L.kvqo_rotate.argtypes = [P, P, C.c_int, P]
        L.kvqo_rotate_f64.argtypes = [P, P, C.c_int, P]
        L.kvqo_page_bytes.argtypes = [C.POINTER(_Layout)] + [C.POINTER(C.c_size_t)] * 4
        L.kvqo_quantize_append.argtypes = [C.POINTER(_Layout), C.POINTER(_Cache), P, P,
                                           C.c_int, P, P]
        L.kvqo_dequantize.argtypes = [C.POINTER(_Layout), C.POINTER(_Cache), P, C.c_int, P, P]
        L.kvqo_attention_dense.argtypes = [P, P, P, C.c_int, C.c_int, C.c_double, P, P]
        L.kvqo_decode_attention.argtypes = [C.POINTER(_Layout), C.POINTER(_Cache), P, C.c_int,
                                            P, C.c_double, P, P]
        L.kvqo_prefill_attention.argtypes = [C.POINTER(_Layout), C.POINTER(_Cache), P, C.c_int,
                                             P, P, C.c_double, P, P]
        L.kvqo_num_threads.restype = C.c_int
        L.kvqo_set_num_threads.argtypes = [C.c_int]
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(C.c_void_p)


# ------------------------------------------------------------ scalar helpers

def f32_to_f16(x, mode=RN) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32).ravel()
    out = np.empty(x.size, dtype=np.uint16)
    lib().kvqo_f32_to_f16_n(_p(x), x.size, mode, _p(out))
    return out


def f32_to_bf16(x, mode=RN) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32).ravel()
    out = np.empty(x.size, dtype=np.uint16)
    lib().kvqo_f32_to_bf16_n(_p(x), x.size, mode, _p(out))
    return out


def f16_to_f32(h) -> np.ndarray:
    h = np.asarray(h, dtype=np.uint16).ravel()
    return np.array([lib().kvqo_f16_to_f32(int(v)) for v in h], dtype=np.float32)


def fp_op(a, b, op: str, up: bool) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float32).ravel()
    b = np.ascontiguousarray(b, dtype=np.float32).ravel()
    out = np.empty(a.size, dtype=np.float32)
    lib().kvqo_op_n(_p(a), _p(b), a.size, 0 if op == "sub" else 1, int(up), _p(out))
    return out


def quantize_rows(x: np.ndarray, group: int, bits: int):
    """x [rows][row_len] fp32 -> (scale u16 [rows][ng], zero u16, codes u8 [rows][row_len])."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    rows, n = x.shape
    ng = n // group
    s = np.empty((rows, ng), np.uint16)
    z = np.empty((rows, ng), np.uint16)
    c = np.empty((rows, n), np.uint8)
    lib().kvqo_quantize_rows(_p(x), rows, n, group, bits, _p(s), _p(z), _p(c))
    return s, z, c


def dequantize_rows(codes, scale, zero, group: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scale = np.ascontiguousarray(scale, dtype=np.uint16)
    zero = np.ascontiguousarray(zero, dtype=np.uint16)
    rows, n = codes.shape
    out = np.empty((rows, n), np.float32)
    lib().kvqo_dequantize_rows(_p(codes), _p(scale), _p(zero), rows, n, group, _p(out))
    return out


def pack(codes, bits: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8).ravel()
    out = np.zeros(((codes.size * bits + 31) // 32) * 4, dtype=np.uint8)
    lib().kvqo_pack(_p(codes), codes.size, bits, _p(out))
    return out


def unpack(packed, n: int, bits: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    return np.array([lib().kvqo_unpack_one(_p(packed), i, bits) for i in range(n)], np.uint8)


def hadamard(n: int) -> np.ndarray:
    H = np.empty((n, n), np.float64)
    lib().kvqo_hadamard(n, _p(H))
    return H


def rotate(x, signs) -> np.ndarray:
    """rows of x (fp32 [..., d]) rotated by sigma-then-Hadamard, rounded to fp32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    signs = np.ascontiguousarray(signs, dtype=np.int8)
    d = x.shape[-1]
    flat = x.reshape(-1, d)
    out = np.empty_like(flat)
    for i in range(flat.shape[0]):
        lib().kvqo_rotate(_p(flat[i]), _p(signs), d, _p(out[i]))
    return out.reshape(x.shape)


def attention_dense(q, K, V, sm_scale: float):
    q = np.ascontiguousarray(q, dtype=np.float64)
    K = np.ascontiguousarray(K, dtype=np.float64)
    V = np.ascontiguousarray(V, dtype=np.float64)
    L, d = K.shape if K.ndim == 2 else (0, q.shape[0])
    o = np.empty(d, np.float64)
    lse = np.empty(1, np.float64)
    lib().kvqo_attention_dense(_p(q), _p(K), _p(V), L, d, float(sm_scale), _p(o), _p(lse))
    return o, float(lse[0])


def num_threads() -> int:
    return int(lib().kvqo_num_threads())


def set_num_threads(n: int) -> None:
    lib().kvqo_set_num_threads(int(n))


# ------------------------------------------------------------ paged cache

@dataclass
class Layout:
    head_dim: int
    num_q_heads: int
    num_kv_heads: int
    k_bits: int = 4
    v_bits: int = 2
    k_group: int = 32
    v_group: int = 128
    page_size: int = 64
    window: int = 0
    rotate_keys: bool = False
    rot_signs: Optional[np.ndarray] = None
    k_per_channel: bool = False        # key groups of k_group positions of one channel

    @classmethod
    def from_workload(cls, w, signs=None):
        return cls(w.head_dim, w.num_q_heads, w.num_kv_heads, w.k_bits, w.v_bits,
                   w.k_group, w.v_group, w.page_size, w.window, bool(w.rotate_keys),
                   signs, bool(getattr(w, "k_per_channel", False)))

    @property
    def ring_slots(self) -> int:
        """bf16 ring rows per (sequence, kv-head): W, plus k_group - 1 when key
        groups run along positions (a group waits there until complete)."""
        return self.window + (self.k_group - 1 if self.k_per_channel else 0)


class Cache:
    """Host-memory cache in the library's storage format, driven by the oracle."""

    def __init__(self, layout: Layout, batch: int, page_table: np.ndarray, num_pages: int):
        self.layout = layout
        self.batch = batch
        self.page_table = np.ascontiguousarray(page_table, dtype=np.int32)
        d, H, P = layout.head_dim, layout.num_kv_heads, layout.page_size
        self.num_pages = num_pages
        self.k_codes = np.zeros((num_pages, H, P, d * layout.k_bits // 8), np.uint8)
        if layout.k_per_channel:
            self.k_meta = np.zeros((num_pages, H, P // layout.k_group, d, 2), np.uint16)
        else:
            self.k_meta = np.zeros((num_pages, H, P, d // layout.k_group, 2), np.uint16)
        self.v_codes = np.zeros((num_pages, H, d, P * layout.v_bits // 8), np.uint8)
        self.v_meta = np.zeros((num_pages, H, P, d // layout.v_group, 2), np.uint16)
        R = max(layout.ring_slots, 0)
        self.k_win = np.zeros((batch, H, max(R, 1), d), np.uint16)
        self.v_win = np.zeros((batch, H, max(R, 1), d), np.uint16)
        self._signs = (np.ascontiguousarray(layout.rot_signs, dtype=np.int8)
                       if layout.rot_signs is not None else None)

    def _structs(self):
        l = self.layout
        lay = _Layout(l.head_dim, l.num_q_heads, l.num_kv_heads, l.k_bits, l.v_bits,
                      l.k_group, l.v_group, l.page_size, l.window, int(l.rotate_keys),
                      _p(self._signs) if self._signs is not None else None, int(l.k_per_channel))
        cache = _Cache(_p(self.k_codes), _p(self.v_codes), _p(self.k_meta), _p(self.v_meta),
                       _p(self.k_win), _p(self.v_win), _p(self.page_table), self.batch,
                       self.page_table.shape[1])
        return lay, cache

    def append(self, k_new, v_new, in_dtype: int, cu_new, lens) -> None:
        lay, cache = self._structs()
        k_new = np.ascontiguousarray(k_new)
        v_new = np.ascontiguousarray(v_new)
        cu = np.ascontiguousarray(cu_new, dtype=np.int32)
        ln = np.ascontiguousarray(lens, dtype=np.int32)
        rc = lib().kvqo_quantize_append(C.byref(lay), C.byref(cache), _p(k_new), _p(v_new),
                                        in_dtype, _p(cu), _p(ln))
        if rc != 0:
            raise ValueError(f"oracle append failed: {rc}")

    def dequantize(self, lens, max_len: int):
        lay, cache = self._structs()
        ln = np.ascontiguousarray(lens, dtype=np.int32)
        d, H = self.layout.head_dim, self.layout.num_kv_heads
        k = np.zeros((self.batch, H, max_len, d), np.float32)
        v = np.zeros((self.batch, H, max_len, d), np.float32)
        rc = lib().kvqo_dequantize(C.byref(lay), C.byref(cache), _p(ln), max_len, _p(k), _p(v))
        if rc != 0:
            raise ValueError(f"oracle dequantize failed: {rc}")
        return k, v

    def decode_attention(self, q, q_dtype: int, lens, sm_scale: float):
        lay, cache = self._structs()
        q = np.ascontiguousarray(q)
        ln = np.ascontiguousarray(lens, dtype=np.int32)
        Hq, d = self.layout.num_q_heads, self.layout.head_dim
        out = np.empty((self.batch, Hq, d), np.float64)
        lse = np.empty((self.batch, Hq), np.float64)
        rc = lib().kvqo_decode_attention(C.byref(lay), C.byref(cache), _p(q), q_dtype, _p(ln),
                                         float(sm_scale), _p(out), _p(lse))
        if rc != 0:
            raise ValueError(f"oracle attention failed: {rc}")
        return out, lse

    def prefill_attention(self, q, q_dtype: int, cu_q, lens, sm_scale: float):
        """Causal attention of a chunk of new queries (rows cu_q[b]..cu_q[b+1]
        of q [total_q][Hq][d]) whose keys and values are the newest positions
        of each sequence; query i of sequence b sees positions
        [0, lens[b] - n_b + i].  Returns out [total_q][Hq][d], lse [total_q][Hq]."""
        lay, cache = self._structs()
        q = np.ascontiguousarray(q)
        cu = np.ascontiguousarray(cu_q, dtype=np.int32)
        ln = np.ascontiguousarray(lens, dtype=np.int32)
        Hq, d = self.layout.num_q_heads, self.layout.head_dim
        total = int(cu[-1])
        out = np.zeros((total, Hq, d), np.float64)
        lse = np.zeros((total, Hq), np.float64)
        rc = lib().kvqo_prefill_attention(C.byref(lay), C.byref(cache), _p(q), q_dtype, _p(cu), _p(ln),
                                          float(sm_scale), _p(out), _p(lse))
        if rc != 0:
            raise ValueError(f"oracle prefill attention failed: {rc}")
        return out, lse


def page_bytes(layout: Layout):
    lay = _Layout(layout.head_dim, layout.num_q_heads, layout.num_kv_heads, layout.k_bits,
                  layout.v_bits, layout.k_group, layout.v_group, layout.page_size,
                  layout.window, int(layout.rotate_keys), None, int(layout.k_per_channel))
    vals = [C.c_size_t() for _ in range(4)]
    rc = lib().kvqo_page_bytes(C.byref(lay), *[C.byref(v) for v in vals])
    if rc != 0:
        raise ValueError(f"unsupported layout: {rc}")
    return tuple(int(v.value) for v in vals)
