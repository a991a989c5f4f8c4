"""The per-channel key-group kernels, run on the CPU, against the oracle.

tests/emu/kernel_emu.cpp runs the CUDA kernels' own CTA bodies
(csrc/kvq_channel_body.cuh for the append and dequantize kernels,
csrc/kvq_prefill_body.cuh for decode and chunked-prefill attention) as host
C++ under AddressSanitizer and UBSan, with the IEEE directed-rounding
operations taken from the C library's rounding modes.  The append must
leave cache bytes identical to the oracle's after every call (prefill,
decode steps, chunks that complete several groups); dequantize must return
the oracle's values exactly; attention must agree within 1e-3 + 1e-3*|ref|.
The GPU parity tests of the same kernels are tests/test_gpu_per_channel.py.
"""
import numpy as np
import pytest

import emu_harness as emu
import oracle
import workloads as wl

ATOL = RTOL = 1e-3
NAMES = ("k_codes", "k_meta", "v_codes", "v_meta", "k_win", "v_win")


@pytest.fixture(scope="module")
def emu_exe(tmp_path_factory):
    exe = emu.build(str(tmp_path_factory.mktemp("emu")))
    if exe is None:
        pytest.skip("g++ or the CUDA headers are missing")
    return exe


BASE = wl.Workload(name="pc_emu", batch=3, num_q_heads=8, num_kv_heads=2, head_dim=64, seq_len=0,
                   k_bits=4, v_bits=2, k_group=32, v_group=64, window=8, k_per_channel=True,
                   ragged=(1, 150), shuffle_pages=True, outliers=("random", 2, 10.0), seed=23)


class EmuCache:
    """Cache arrays driven by the emulated append kernels, beside an oracle cache."""

    def __init__(self, exe, tmp, w, capacity):
        self.exe, self.tmp, self.w = exe, tmp, w
        pt = wl.page_table(w, np.maximum(0, np.asarray(capacity) - w.window))
        self.oc = oracle.Cache(oracle.Layout.from_workload(w), w.batch, pt, max(1, int((pt >= 0).sum())))
        self.arr = {n: np.zeros_like(getattr(self.oc, n)) for n in NAMES}
        self.lens = np.zeros(w.batch, np.int32)

    def append(self, k, v, cu):
        w = self.w
        params, arrays = emu.cache_params(self.oc)
        arrays.update(self.arr)
        n = np.diff(cu)
        params.update(mode=emu.MODE_APPEND_PC, in_bf16=int(w.in_dtype == wl.DT_BF16), max_new=int(n.max()))
        arrays.update(k_new=k, v_new=v, cu_new=np.asarray(cu, np.int32), lens=self.lens)
        out = emu.run(self.exe, self.tmp, params, arrays,
                      {n_: (self.arr[n_].dtype, self.arr[n_].shape) for n_ in NAMES})
        self.arr.update(out)
        dt = oracle.IN_BF16 if w.in_dtype == wl.DT_BF16 else oracle.IN_F32
        self.oc.append(k, v, dt, cu, self.lens)
        self.lens = self.lens + n.astype(np.int32)

    def compare(self):
        for n in NAMES:
            got, want = self.arr[n], getattr(self.oc, n)
            if not np.array_equal(got, want):
                bad = np.flatnonzero(got.view(np.uint8).ravel() != want.view(np.uint8).ravel())
                raise AssertionError(f"{n}: {bad.size} bytes differ, first at {bad[:8]}")

    def view_params(self):
        params, arrays = emu.cache_params(self.oc)
        arrays.update(self.arr)
        return params, arrays


def _chunk_rows(w, start, n):
    ks, vs = [], []
    for b in range(w.batch):
        if n[b]:
            kr, vr, _, _ = wl.seq_kv(w, b, int(n[b]), start=int(start[b]))
            ks.append(kr)
            vs.append(vr)
    return np.concatenate(ks), np.concatenate(vs)


CASES = {
    "d64_k4v2_g32_w8": dict(),
    "d64_k4v2_g16_w0": dict(k_group=16, window=0),
    "d128_k2v4_g64_w40": dict(head_dim=128, k_bits=2, v_bits=4, k_group=64, v_group=128, window=40),
    "d64_k1v1_g16_w8_f32": dict(k_bits=1, v_bits=1, k_group=16, v_group=32, in_dtype=wl.DT_F32),
    "d64_k8v8_g32_w3": dict(k_bits=8, v_bits=8, window=3),
}


@pytest.mark.parametrize("name", list(CASES))
def test_emulated_append_bit_exact(emu_exe, tmp_path, name):
    """Prefill, then single-token decode steps, then a chunk that completes
    several groups; cache bytes equal the oracle's after every call."""
    w = BASE.with_(**CASES[name])
    lens0 = wl.lengths(w)
    lens0[0] = 0
    steps, chunk = 20, 70
    ec = EmuCache(emu_exe, str(tmp_path), w, lens0 + steps + chunk)
    kr, vr, _, _, cu, _ = wl.prefill(w, lens0, with_f32=False)
    ec.append(kr, vr, cu)
    ec.compare()
    ones = np.arange(w.batch + 1, dtype=np.int32)
    for s in range(steps):
        k, v = _chunk_rows(w, ec.lens, np.ones(w.batch, np.int32))
        ec.append(k, v, ones)
        if s % 5 == 4:
            ec.compare()
    n = np.array([chunk, 1, 33][:w.batch], np.int32)
    k, v = _chunk_rows(w, ec.lens, n)
    ec.append(k, v, np.concatenate([[0], np.cumsum(n)]).astype(np.int32))
    ec.compare()


def test_emulated_dequantize_and_attention(emu_exe, tmp_path):
    w = BASE.with_(head_dim=128, v_group=128, k_group=32, window=16)
    lens0 = wl.lengths(w)
    lens0[2] = 0
    ec = EmuCache(emu_exe, str(tmp_path), w, lens0)
    kr, vr, _, _, cu, _ = wl.prefill(w, lens0, with_f32=False)
    ec.append(kr, vr, cu)
    lens = ec.lens
    max_len = int(lens.max())
    # dequantize
    params, arrays = ec.view_params()
    params.update(mode=emu.MODE_DEQUANT_PC, max_len=max_len)
    arrays.update(lens=lens)
    shape = (w.batch, w.num_kv_heads, max_len, w.head_dim)
    r = emu.run(emu_exe, str(tmp_path), params, arrays, {"k_out": (np.float32, shape), "v_out": (np.float32, shape)})
    kh, vh = ec.oc.dequantize(lens, max_len)
    for b in range(w.batch):
        L = int(lens[b])
        np.testing.assert_array_equal(r["k_out"][b, :, :L], kh[b, :, :L])
        np.testing.assert_array_equal(r["v_out"][b, :, :L], vh[b, :, :L])
    sc = 1 / np.sqrt(w.head_dim)
    # decode: one query per sequence through the attention body
    q, _ = wl.query(w)
    params, arrays = ec.view_params()
    params.update(mode=emu.MODE_ATTENTION, q_bf16=1, one_query=1, max_q=1, len_cap=max_len, sm_scale=sc)
    arrays.update(q=q, lens=lens)
    r = emu.run(emu_exe, str(tmp_path), params, arrays,
                {"out": (np.float32, (w.batch, w.num_q_heads, w.head_dim)),
                 "lse": (np.float32, (w.batch, w.num_q_heads))})
    ref, ref_lse = ec.oc.decode_attention(q, oracle.IN_BF16, lens, sc)
    np.testing.assert_allclose(r["out"], ref, atol=ATOL, rtol=RTOL)
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(r["lse"]), fin)
    np.testing.assert_allclose(r["lse"][fin], ref_lse[fin], atol=ATOL, rtol=RTOL)
    assert np.all(r["out"][2] == 0)
    # chunked prefill over the same cache
    n = np.minimum(lens, 45).astype(np.int32)
    cu_q = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    qc, _ = wl.chunk_queries(w, int(cu_q[-1]))
    params, arrays = ec.view_params()
    params.update(mode=emu.MODE_ATTENTION, q_bf16=1, one_query=0, max_q=int(n.max()), sm_scale=sc)
    arrays.update(q=qc, cu_q=cu_q, lens=lens)
    r = emu.run(emu_exe, str(tmp_path), params, arrays,
                {"out": (np.float32, (int(cu_q[-1]), w.num_q_heads, w.head_dim)),
                 "lse": (np.float32, (int(cu_q[-1]), w.num_q_heads))})
    ref, ref_lse = ec.oc.prefill_attention(qc, oracle.IN_BF16, cu_q, lens, sc)
    np.testing.assert_allclose(r["out"], ref, atol=ATOL, rtol=RTOL)
    np.testing.assert_allclose(r["lse"], ref_lse, atol=ATOL, rtol=RTOL)


@pytest.mark.parametrize("seed", range(10))
def test_emulated_append_random_sequences(emu_exe, tmp_path, seed):
    """Random per-channel layouts and random append sizes (0 to 69 tokens per
    sequence per call); bytes equal the oracle's after every call."""
    r = np.random.default_rng([seed, 78])
    d = int(r.choice([64, 128]))
    hkv = int(r.choice([1, 2]))
    w = wl.Workload(name="random", batch=int(r.integers(1, 4)), num_q_heads=2 * hkv, num_kv_heads=hkv, head_dim=d,
                    seq_len=0, k_bits=int(r.choice([1, 2, 4, 8])), v_bits=int(r.choice([1, 2, 4, 8])),
                    k_group=int(r.choice([16, 32, 64])), v_group=int(r.choice([x for x in (16, 32, 64, 128) if x <= d])),
                    window=int(r.choice([0, 1, 7, 16, 64, 100])), k_per_channel=True,
                    ragged=(0, int(r.integers(1, 200))), shuffle_pages=True, outliers=("random", 1, 10.0),
                    seed=int(r.integers(0, 1 << 30)), in_dtype=wl.DT_BF16 if r.integers(0, 3) else wl.DT_F32)
    lens0 = wl.lengths(w)
    steps = [r.integers(0, 70, w.batch).astype(np.int32) for _ in range(3)]
    ec = EmuCache(emu_exe, str(tmp_path), w, lens0 + sum(steps))
    kr, vr, _, _, cu, _ = wl.prefill(w, lens0, with_f32=False)
    if cu[-1] > 0:
        ec.append(kr, vr, cu)
        ec.compare()
    for n in steps:
        if n.sum() == 0:
            continue
        k, v = _chunk_rows(w, ec.lens, n)
        ec.append(k, v, np.concatenate([[0], np.cumsum(n)]).astype(np.int32))
        ec.compare()
