"""Helpers for the GPU parity tests: the same seeded inputs drive the CUDA
library (through its C ABI) and the CPU oracle, and their outputs are
compared.  No expected value comes from the CUDA side."""
from __future__ import annotations

import os

import numpy as np
import torch

import mixed_precision_quantized_kvq_b200 as kvq
import oracle
import workloads as wl

# attention tolerance against the fp64 oracle on the same reconstructed cache
ATOL = 1e-3
RTOL = 1e-3


def torch_raw(a: np.ndarray, device="cuda") -> torch.Tensor:
    """bf16 bit patterns (uint16) or fp32 numpy -> device tensor of that dtype."""
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def in_code(w) -> int:
    return oracle.IN_BF16 if w.in_dtype == wl.DT_BF16 else oracle.IN_F32


class Pair:
    """A GPU cache and an oracle cache with the same layout and page table."""

    def __init__(self, w: wl.Workload, lens: np.ndarray, steps: int = 0, device="cuda"):
        self.w = w
        self.device = device
        self.lens = np.asarray(lens, np.int32).copy()
        cap = np.maximum(0, self.lens + steps - w.window)
        self.pt = wl.page_table(w, cap)
        self.num_pages = max(1, int((self.pt >= 0).sum()))
        self.signs = wl.rotation_signs(w) if w.rotate_keys else None
        self.olay = oracle.Layout.from_workload(w, self.signs)
        self.ocache = oracle.Cache(self.olay, w.batch, self.pt, self.num_pages)
        self.glay = kvq.Layout(w.head_dim, w.num_q_heads, w.num_kv_heads, w.k_bits, w.v_bits,
                               w.k_group, w.v_group, w.page_size, w.window, w.rotate_keys,
                               torch.from_numpy(self.signs).to(device) if self.signs is not None else None,
                               w.k_per_channel)
        self.gcache = kvq.PagedCache.allocate(self.glay, torch.from_numpy(self.pt).to(device),
                                              self.num_pages)
        self.glens = torch.from_numpy(self.lens).to(device)

    # ---------------------------------------------------------------- append
    def append(self, k_raw, v_raw, cu, oracle_k=None, oracle_dtype=None):
        """Append rows to both caches (oracle_k overrides the oracle's key rows)."""
        n = np.diff(cu)
        max_new = int(n.max()) if n.size else 0
        kvq.kvq_quantize_append(self.glay, self.gcache, torch_raw(k_raw, self.device),
                                torch_raw(v_raw, self.device),
                                torch.from_numpy(np.asarray(cu, np.int32)).to(self.device),
                                self.glens, max_new)
        ok = k_raw if oracle_k is None else oracle_k
        ov = v_raw
        dt = in_code(self.w) if oracle_dtype is None else oracle_dtype
        if oracle_dtype == oracle.IN_F32 and v_raw.dtype == np.uint16:
            ov = wl.bf16_to_f32(v_raw)
        self.ocache.append(ok, ov, dt, cu, self.lens)
        self.lens = self.lens + n.astype(np.int32)
        self.glens += torch.from_numpy(n.astype(np.int32)).to(self.device)

    def prefill(self, with_f32: bool = True):
        kr, vr, kf, vf, cu, _ = wl.prefill(self.w, self.lens, with_f32=with_f32)
        self.lens[:] = 0
        self.glens.zero_()
        self.append(kr, vr, cu)
        return kr, vr, kf, vf, cu

    # ---------------------------------------------------------------- compare
    def gpu_bytes(self, name: str) -> np.ndarray:
        t = getattr(self.gcache, name)
        return t.cpu().numpy().view(np.uint8)

    def compare_cache(self):
        """Codes, metadata and window are bit-identical to the oracle's."""
        names = ["k_codes", "k_meta", "v_codes", "v_meta"]
        if self.olay.ring_slots > 0:
            names += ["k_win", "v_win"]
        for name in names:
            want = getattr(self.ocache, name).view(np.uint8).ravel()
            got = self.gpu_bytes(name)[: want.size]
            if not np.array_equal(got, want):
                bad = np.flatnonzero(got != want)
                raise AssertionError(f"{name}: {bad.size} bytes differ, first at {bad[:8]} "
                                     f"(gpu {got[bad[:8]]}, oracle {want[bad[:8]]})")

    def decode(self, step: int = 0, max_len=None):
        qr, qf = wl.query(self.w, step)
        max_len = int(self.lens.max()) if max_len is None else max_len
        out, lse = kvq.decode_attention(self.glay, self.gcache, torch_raw(qr, self.device),
                                        self.glens, max_len, 1.0 / np.sqrt(self.w.head_dim))
        return qr, out.cpu().numpy(), lse.cpu().numpy()

    def oracle_decode(self, qr, rows=None):
        return self.ocache.decode_attention(qr, in_code(self.w), self.lens,
                                            1.0 / np.sqrt(self.w.head_dim))

    def check_decode(self, step: int = 0):
        qr, out, lse = self.decode(step)
        ref, ref_lse = self.oracle_decode(qr)
        log = os.environ.get("KVQ_PARITY_LOG")
        if log:                                   # optional record of the errors (max abs, max rel)
            err = np.abs(np.asarray(out, np.float64) - ref)
            rel = err / np.maximum(np.abs(ref), 1e-30)
            with open(log, "a") as f:
                f.write(f"{os.environ.get('PYTEST_CURRENT_TEST', '?').split(' ')[0]} step {step}: "
                        f"max_abs {err.max() if err.size else 0.0:.3e} "
                        f"max_rel(|ref|>1e-2) {rel[np.abs(ref) > 1e-2].max() if (np.abs(ref) > 1e-2).any() else 0.0:.3e}\n")
        check_close(out, ref, "out")
        finite = np.isfinite(ref_lse)
        assert np.array_equal(np.isfinite(lse), finite)
        check_close(lse[finite], ref_lse[finite], "lse")
        return out, ref

    def dequantize(self, max_len=None):
        max_len = int(self.lens.max()) if max_len is None else max_len
        shape = (self.w.batch, self.w.num_kv_heads, max_len, self.w.head_dim)
        k = torch.zeros(shape, dtype=torch.float32, device=self.device)
        v = torch.zeros(shape, dtype=torch.float32, device=self.device)
        kvq.kvq_dequantize(self.glay, self.gcache, self.glens, max_len, k, v)
        return k.cpu().numpy(), v.cpu().numpy()


    def check_dequantize(self, max_len=None):
        """kvq_dequantize is bit-identical to the oracle's reconstruction:
        code*scale+zero in one fp32 fma for quantized positions (keys in the
        rotated domain when the layout rotates them), widened bf16 for window
        positions; positions at or past a sequence's length are not written
        (zeros here)."""
        max_len = int(self.lens.max()) if max_len is None else max_len
        k, v = self.dequantize(max_len)
        ko, vo = self.ocache.dequantize(self.lens, max_len)
        for name, got, want in (("keys", k, ko), ("values", v, vo)):
            for b in range(self.w.batch):
                L = int(min(self.lens[b], max_len))
                g, o = got[b, :, :L], want[b, :, :L]
                if not np.array_equal(g.view(np.uint32), o.view(np.uint32)):
                    bad = np.argwhere(g.view(np.uint32) != o.view(np.uint32))
                    raise AssertionError(f"{name} of sequence {b}: {len(bad)} values differ, first {bad[:4].tolist()}")
                assert not got[b, :, L:].any(), f"{name} of sequence {b} written past its length"


def check_close(got, want, what="value"):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape
    if got.size == 0:
        return 0.0
    err = np.abs(got - want)
    lim = ATOL + RTOL * np.abs(want)
    if not np.all(err <= lim):
        i = np.unravel_index(np.argmax(err - lim), err.shape)
        raise AssertionError(f"{what}: max err {err.max():.3e}, worst at {i}: got {got[i]!r} want {want[i]!r}")
    return float(err.max())
