"""Python binding of the B200 quantized KV-cache library (``libkvq.so``).

Argument marshalling only: every step of quantization and attention runs in
the library's CUDA kernels; PyTorch provides device memory and streams.  The
functions carry the names of the C ABI in ``include/kvq.h``.  There is no CPU
fallback: if ``libkvq.so`` is missing, loading raises.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass, field
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkvq.so")

KVQ_OK = 0
KVQ_ERR_INVALID_ARG = -1
KVQ_ERR_UNSUPPORTED = -2
KVQ_ERR_WORKSPACE = -3
KVQ_ERR_CUDA = -4
KVQ_F32 = 0
KVQ_BF16 = 1
KVQ_STATIC_SCRATCH_BYTES = 16 * 1024 * 1024
PAGE_SIZE = 64


class KVQError(RuntimeError):
    def __init__(self, call: str, status: int):
        super().__init__(f"{call}: {kvq_status_string(status)} (status {status})")
        self.status = status


class kvq_layout(C.Structure):
    _fields_ = [("head_dim", C.c_int), ("num_q_heads", C.c_int), ("num_kv_heads", C.c_int),
                ("k_bits", C.c_int), ("v_bits", C.c_int), ("k_group", C.c_int),
                ("v_group", C.c_int), ("page_size", C.c_int), ("window", C.c_int),
                ("rotate_keys", C.c_int), ("rot_signs", C.c_void_p), ("k_per_channel", C.c_int)]


class kvq_cache(C.Structure):
    _fields_ = [("k_codes", C.c_void_p), ("v_codes", C.c_void_p), ("k_meta", C.c_void_p),
                ("v_meta", C.c_void_p), ("k_win", C.c_void_p), ("v_win", C.c_void_p),
                ("page_table", C.c_void_p), ("batch", C.c_int),
                ("max_pages_per_seq", C.c_int), ("num_pages", C.c_int)]


_lib_handle = None


def lib() -> C.CDLL:
    """Load libkvq.so (raises if it has not been built)."""
    global _lib_handle
    if _lib_handle is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} not found: build it with "
                              "`python -m mixed_precision_quantized_kvq_b200.build`")
        L = C.CDLL(LIB_PATH)
        P, I, S = C.c_void_p, C.c_int, C.c_size_t
        LP, CP = C.POINTER(kvq_layout), C.POINTER(kvq_cache)
        L.kvq_status_string.restype = C.c_char_p
        L.kvq_status_string.argtypes = [I]
        L.kvq_version.restype = I
        L.kvq_page_bytes.argtypes = [LP] + [C.POINTER(S)] * 4
        L.kvq_window_bytes.argtypes = [LP, I, C.POINTER(S)]
        L.kvq_decode_workspace_bytes.restype = S
        L.kvq_decode_workspace_bytes.argtypes = [LP, I, I]
        L.kvq_quantize_append.argtypes = [LP, CP, P, P, I, P, P, I, P]
        L.kvq_decode_attention.argtypes = [LP, CP, P, I, P, I, C.c_float, P, P, P, S, P]
        L.kvq_decode_attention_static_scratch.argtypes = [LP, CP, P, I, P, I, C.c_float, P, P, P]
        L.kvq_append_decode.argtypes = [LP, CP, P, P, I, P, P, I, P, I, P, I, C.c_float, P, P, P, S, P]
        L.kvq_dequantize.argtypes = [LP, CP, P, I, P, P, P]
        L.kvq_prefill_attention.argtypes = [LP, CP, P, I, P, P, I, C.c_float, P, P, P]
        L.kvq_rotate_keys.argtypes = [LP, P, I, I, P, P]
        L.kvq_set_decode_path.argtypes = [I]
        L.kvq_set_decode_path.restype = I
        L.kvq_get_decode_path.argtypes = [LP]
        L.kvq_get_decode_path.restype = I
        L.kvq_decode_status.argtypes = [C.POINTER(C.c_uint), C.POINTER(C.c_uint), I]
        L.kvq_decode_status.restype = I
        for n in ("kvq_page_bytes", "kvq_window_bytes", "kvq_quantize_append",
                  "kvq_decode_attention", "kvq_decode_attention_static_scratch", "kvq_append_decode",
                  "kvq_dequantize",
                  "kvq_rotate_keys"):
            getattr(L, n).restype = I
        _lib_handle = L
    return _lib_handle


def kvq_status_string(status: int) -> str:
    return lib().kvq_status_string(int(status)).decode()


def kvq_version() -> int:
    return int(lib().kvq_version())


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return C.c_void_p(t.data_ptr())


def _check(t: Optional[torch.Tensor], name: str, dtypes, numel: Optional[int] = None,
           at_least: bool = False, optional: bool = False) -> None:
    """Argument checks before a C call: a CUDA tensor on the current device,
    contiguous, of one of `dtypes`, with exactly (or at least) `numel`
    elements.  A wrong buffer would otherwise be read or written past its end
    by a kernel."""
    if t is None:
        if optional:
            return
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor):
        raise ValueError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor, got {t.device}")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name} is on {t.device}, not on the current CUDA device "
                         f"cuda:{torch.cuda.current_device()}")
    if t.dtype not in dtypes:
        raise ValueError(f"{name} must have dtype {' or '.join(str(d) for d in dtypes)}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if numel is not None:
        n = t.numel()
        if (n < numel) if at_least else (n != numel):
            raise ValueError(f"{name} has {n} elements, expected {'at least ' if at_least else ''}{numel}")


_FLOAT_IN = (torch.bfloat16, torch.float32)
_I32 = (torch.int32,)
_F32 = (torch.float32,)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KVQ_BF16
    if t.dtype == torch.float32:
        return KVQ_F32
    raise ValueError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _stream(stream) -> C.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _call(name: str, *args) -> None:
    rc = getattr(lib(), name)(*args)
    if rc != KVQ_OK:
        raise KVQError(name, rc)


@dataclass
class Layout:
    head_dim: int
    num_q_heads: int
    num_kv_heads: int
    k_bits: int = 4
    v_bits: int = 2
    k_group: int = 32
    v_group: int = 128
    page_size: int = PAGE_SIZE
    window: int = 0
    rotate_keys: bool = False
    rot_signs: Optional[torch.Tensor] = None     # device int8 [head_dim]
    k_per_channel: bool = False                  # key groups of k_group positions of one channel

    def c(self) -> kvq_layout:
        return kvq_layout(self.head_dim, self.num_q_heads, self.num_kv_heads, self.k_bits,
                          self.v_bits, self.k_group, self.v_group, self.page_size, self.window,
                          int(self.rotate_keys), _ptr(self.rot_signs), int(self.k_per_channel))


@dataclass
class PagedCache:
    """Device buffers of one layer's cache in the layout kvq.h documents."""
    k_codes: torch.Tensor
    v_codes: torch.Tensor
    k_meta: torch.Tensor
    v_meta: torch.Tensor
    k_win: Optional[torch.Tensor]
    v_win: Optional[torch.Tensor]
    page_table: torch.Tensor                      # int32 [batch][max_pages]
    num_pages: int

    @property
    def batch(self) -> int:
        return int(self.page_table.shape[0])

    @classmethod
    def allocate(cls, layout: Layout, page_table: torch.Tensor, num_pages: int) -> "PagedCache":
        dev = page_table.device
        kc, km, vc, vm = kvq_page_bytes(layout)
        batch = int(page_table.shape[0])
        wb = kvq_window_bytes(layout, batch)
        z = lambda n: torch.zeros(max(int(n), 16), dtype=torch.uint8, device=dev)
        win = (z(wb), z(wb)) if wb > 0 else (None, None)
        return cls(z(kc * num_pages), z(vc * num_pages), z(km * num_pages), z(vm * num_pages),
                   win[0], win[1], page_table.to(torch.int32).contiguous(), num_pages)

    def c(self) -> kvq_cache:
        return kvq_cache(_ptr(self.k_codes), _ptr(self.v_codes), _ptr(self.k_meta),
                         _ptr(self.v_meta), _ptr(self.k_win), _ptr(self.v_win),
                         _ptr(self.page_table), self.batch, int(self.page_table.shape[1]),
                         int(self.num_pages))


def kvq_page_bytes(layout: Layout) -> Tuple[int, int, int, int]:
    vals = [C.c_size_t() for _ in range(4)]
    _call("kvq_page_bytes", C.byref(layout.c()), *[C.byref(v) for v in vals])
    return tuple(int(v.value) for v in vals)


def kvq_window_bytes(layout: Layout, batch: int) -> int:
    v = C.c_size_t()
    _call("kvq_window_bytes", C.byref(layout.c()), int(batch), C.byref(v))
    return int(v.value)


def kvq_decode_workspace_bytes(layout: Layout, batch: int, max_len: int) -> int:
    return int(lib().kvq_decode_workspace_bytes(C.byref(layout.c()), int(batch), int(max_len)))


def kvq_quantize_append(layout: Layout, cache: PagedCache, k_new: torch.Tensor, v_new: torch.Tensor,
                        cu_new: torch.Tensor, lens: torch.Tensor, max_new: int, stream=None) -> None:
    """kvq.h kvq_quantize_append: k_new/v_new [total_new][Hkv][d] (bf16 or fp32)."""
    if k_new.dtype != v_new.dtype:
        raise ValueError("k_new and v_new must share a dtype")
    B, row = cache.batch, layout.num_kv_heads * layout.head_dim
    _check(k_new, "k_new", _FLOAT_IN)
    if k_new.numel() % row:
        raise ValueError(f"k_new must hold whole rows of {row} elements ([total_new][Hkv][d])")
    _check(v_new, "v_new", _FLOAT_IN, k_new.numel())
    _check(cu_new, "cu_new", _I32, B + 1)
    _check(lens, "lens", _I32, B)
    _call("kvq_quantize_append", C.byref(layout.c()), C.byref(cache.c()), _ptr(k_new), _ptr(v_new),
          _dtype_code(k_new), _ptr(cu_new), _ptr(lens), int(max_new), _stream(stream))


def _nbytes(t: Optional[torch.Tensor]) -> int:
    return 0 if t is None else t.numel() * t.element_size()


def _check_workspace(layout, cache, max_len, workspace):
    """At least kvq_decode_workspace_bytes; optional for key groups along
    positions (without it, or with less, the pairs are not split between CTAs)."""
    if layout.k_per_channel:
        _check(workspace, "workspace", (torch.uint8,), optional=True)
    else:
        _check(workspace, "workspace", (torch.uint8,), kvq_decode_workspace_bytes(layout, cache.batch, max_len),
               at_least=True)


def _check_decode_args(layout, cache, q, lens, out, lse):
    B, Hq, d = cache.batch, layout.num_q_heads, layout.head_dim
    _check(q, "q", _FLOAT_IN, B * Hq * d)
    _check(lens, "lens", _I32, B)
    _check(out, "out", _F32, B * Hq * d)
    _check(lse, "lse", _F32, B * Hq, optional=True)


def kvq_decode_attention(layout: Layout, cache: PagedCache, q: torch.Tensor, lens: torch.Tensor,
                         max_len: int, sm_scale: float, out: torch.Tensor,
                         lse: Optional[torch.Tensor], workspace: torch.Tensor, stream=None) -> None:
    """kvq.h kvq_decode_attention: q [B][Hq][d] -> out fp32 [B][Hq][d], lse fp32 [B][Hq]."""
    _check_decode_args(layout, cache, q, lens, out, lse)
    _check_workspace(layout, cache, max_len, workspace)
    _call("kvq_decode_attention", C.byref(layout.c()), C.byref(cache.c()), _ptr(q), _dtype_code(q),
          _ptr(lens), int(max_len), C.c_float(sm_scale), _ptr(out), _ptr(lse), _ptr(workspace),
          C.c_size_t(_nbytes(workspace)), _stream(stream))


def kvq_append_decode(layout: Layout, cache: PagedCache, k_new: torch.Tensor, v_new: torch.Tensor,
                      cu_new: torch.Tensor, lens_old: torch.Tensor, max_new: int, q: torch.Tensor,
                      lens: torch.Tensor, max_len: int, sm_scale: float, out: torch.Tensor,
                      lse: Optional[torch.Tensor], workspace: torch.Tensor, stream=None) -> None:
    """kvq.h kvq_append_decode: kvq_quantize_append then kvq_decode_attention,
    the decode's start-up overlapping the append."""
    if k_new.dtype != v_new.dtype:
        raise ValueError("k_new and v_new must share a dtype")
    B, row = cache.batch, layout.num_kv_heads * layout.head_dim
    _check(k_new, "k_new", _FLOAT_IN)
    if k_new.numel() % row:
        raise ValueError(f"k_new must hold whole rows of {row} elements ([total_new][Hkv][d])")
    _check(v_new, "v_new", _FLOAT_IN, k_new.numel())
    _check(cu_new, "cu_new", _I32, B + 1)
    _check(lens_old, "lens_old", _I32, B)
    _check_decode_args(layout, cache, q, lens, out, lse)
    _check_workspace(layout, cache, max_len, workspace)
    _call("kvq_append_decode", C.byref(layout.c()), C.byref(cache.c()), _ptr(k_new), _ptr(v_new),
          _dtype_code(k_new), _ptr(cu_new), _ptr(lens_old), int(max_new), _ptr(q), _dtype_code(q), _ptr(lens),
          int(max_len), C.c_float(sm_scale), _ptr(out), _ptr(lse), _ptr(workspace),
          C.c_size_t(_nbytes(workspace)), _stream(stream))


def kvq_decode_attention_static_scratch(layout: Layout, cache: PagedCache, q: torch.Tensor,
                                        lens: torch.Tensor, max_len: int, sm_scale: float,
                                        out: torch.Tensor, lse: Optional[torch.Tensor],
                                        stream=None) -> None:
    """kvq.h kvq_decode_attention_static_scratch: kvq_decode_attention with the
    library's static per-device scratch (KVQ_STATIC_SCRATCH_BYTES) instead of a
    workspace; calls overlapping on the GPU race on that scratch."""
    _check_decode_args(layout, cache, q, lens, out, lse)
    _call("kvq_decode_attention_static_scratch", C.byref(layout.c()), C.byref(cache.c()), _ptr(q),
          _dtype_code(q), _ptr(lens), int(max_len), C.c_float(sm_scale), _ptr(out), _ptr(lse),
          _stream(stream))


def kvq_prefill_attention(layout: Layout, cache: PagedCache, q: torch.Tensor, cu_q: torch.Tensor,
                          lens: torch.Tensor, max_q: int, sm_scale: float, out: torch.Tensor,
                          lse: Optional[torch.Tensor], stream=None) -> None:
    """kvq.h kvq_prefill_attention: causal attention of each sequence's chunk
    of new queries (rows cu_q[b]..cu_q[b+1] of q [total_q][Hq][d]), whose keys
    and values are already appended, -> out fp32 [total_q][Hq][d], lse fp32."""
    B, Hq, d = cache.batch, layout.num_q_heads, layout.head_dim
    _check(q, "q", _FLOAT_IN)
    if q.numel() % (Hq * d):
        raise ValueError(f"q must hold whole rows of {Hq * d} elements ([total_q][Hq][d])")
    T = q.numel() // (Hq * d)
    _check(cu_q, "cu_q", _I32, B + 1)
    _check(lens, "lens", _I32, B)
    _check(out, "out", _F32, T * Hq * d)
    _check(lse, "lse", _F32, T * Hq, optional=True)
    _call("kvq_prefill_attention", C.byref(layout.c()), C.byref(cache.c()), _ptr(q), _dtype_code(q),
          _ptr(cu_q), _ptr(lens), int(max_q), C.c_float(sm_scale), _ptr(out), _ptr(lse), _stream(stream))


def kvq_dequantize(layout: Layout, cache: PagedCache, lens: torch.Tensor, max_len: int,
                   k_out: torch.Tensor, v_out: torch.Tensor, stream=None) -> None:
    """kvq.h kvq_dequantize: fp32 [B][Hkv][max_len][d] reconstructions."""
    n = cache.batch * layout.num_kv_heads * int(max_len) * layout.head_dim
    _check(lens, "lens", _I32, cache.batch)
    _check(k_out, "k_out", _F32, n)
    _check(v_out, "v_out", _F32, n)
    _call("kvq_dequantize", C.byref(layout.c()), C.byref(cache.c()), _ptr(lens), int(max_len),
          _ptr(k_out), _ptr(v_out), _stream(stream))


def kvq_rotate_keys(layout: Layout, k: torch.Tensor, out: torch.Tensor, stream=None) -> None:
    """kvq.h kvq_rotate_keys: rows [rows][d] -> fp32 rotated rows."""
    _check(k, "k", _FLOAT_IN)
    if k.numel() % layout.head_dim:
        raise ValueError(f"k must hold whole rows of {layout.head_dim} elements")
    rows = k.numel() // layout.head_dim
    _check(out, "out", _F32, rows * layout.head_dim)
    _call("kvq_rotate_keys", C.byref(layout.c()), _ptr(k), _dtype_code(k), int(rows), _ptr(out),
          _stream(stream))


DECODE_AUTO, DECODE_CUDA_CORES, DECODE_TENSOR_CORES, DECODE_TCGEN05 = 0, 1, 2, 3
DECODE_PER_CHANNEL = 4   # reported by kvq_get_decode_path for key groups along positions


def kvq_set_decode_path(path: int) -> None:
    """kvq.h kvq_set_decode_path: 0 automatic, 1 CUDA cores, 2 tensor cores
    (persistent kernel), 3 the two-phase tcgen05 kernel."""
    _call("kvq_set_decode_path", int(path))


def kvq_decode_status(clear: bool = False) -> Tuple[int, int]:
    """kvq.h kvq_decode_status: (expired bounded waits, bad merge tickets) on
    the current device; blocking."""
    t, b = C.c_uint(), C.c_uint()
    _call("kvq_decode_status", C.byref(t), C.byref(b), int(bool(clear)))
    return int(t.value), int(b.value)


def kvq_get_decode_path(layout: Layout) -> int:
    rc = int(lib().kvq_get_decode_path(C.byref(layout.c())))
    if rc < 0:
        raise KVQError("kvq_get_decode_path", rc)
    return rc


# ---------------------------------------------------------------- helpers

def workspace_for(layout: Layout, batch: int, max_len: int, device) -> torch.Tensor:
    """A decode workspace, zero-filled as kvq_decode_attention requires before
    its first use (each call leaves it ready for the next)."""
    n = max(kvq_decode_workspace_bytes(layout, batch, max_len), 256)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def decode_attention(layout: Layout, cache: PagedCache, q: torch.Tensor, lens: torch.Tensor,
                     max_len: int, sm_scale: Optional[float] = None,
                     workspace: Optional[torch.Tensor] = None, want_lse: bool = True):
    """Allocating convenience wrapper around kvq_decode_attention."""
    B, Hq, d = q.shape
    if sm_scale is None:
        sm_scale = d ** -0.5
    out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device) if want_lse else None
    if workspace is None:
        workspace = workspace_for(layout, B, max_len, q.device)
    kvq_decode_attention(layout, cache, q, lens, max_len, sm_scale, out, lse, workspace)
    return out, lse


def prefill_attention(layout: Layout, cache: PagedCache, q: torch.Tensor, cu_q: torch.Tensor,
                      lens: torch.Tensor, max_q: int, sm_scale: Optional[float] = None,
                      want_lse: bool = True):
    """Allocating convenience wrapper around kvq_prefill_attention."""
    T, Hq, d = q.shape
    if sm_scale is None:
        sm_scale = d ** -0.5
    out = torch.empty((T, Hq, d), dtype=torch.float32, device=q.device)
    lse = torch.empty((T, Hq), dtype=torch.float32, device=q.device) if want_lse else None
    kvq_prefill_attention(layout, cache, q, cu_q, lens, max_q, sm_scale, out, lse)
    return out, lse


__all__ = [n for n in dir() if n.startswith("kvq_")] + [
    "Layout", "PagedCache", "KVQError", "lib", "decode_attention", "prefill_attention", "workspace_for",
    "LIB_PATH"]
