"""The chunked-prefill kernel body, run on the CPU, against the oracle.

tests/emu/kernel_emu.cpp (driven by tests/emu_harness.py) runs the CUDA
kernel's own per-CTA body (csrc/kvq_prefill_body.cuh) as host C++: one thread per CUDA thread, real
barriers, the GPU's warp-butterfly order.  It is built with AddressSanitizer
and UndefinedBehaviorSanitizer and reads the oracle's cache arrays (the
library's storage format) from exact-size allocations, so these tests check
the kernel's indexing, masking and online softmax, and that it stays inside
every buffer, before it runs on a GPU.  They are not the GPU parity tests
(tests/test_gpu_prefill.py): the emulator is neither the oracle nor a
fallback of the library.
"""
import numpy as np
import pytest

import emu_harness as emu
import oracle
import workloads as wl

ATOL = RTOL = 1e-3


@pytest.fixture(scope="module")
def emu_exe(tmp_path_factory):
    exe = emu.build(str(tmp_path_factory.mktemp("emu")))
    if exe is None:
        pytest.skip("g++ or the CUDA headers are missing")
    return exe


def _run(exe, tmp, c: oracle.Cache, q, q_bf16, cu_q, lens, max_q, sm_scale, signs=None):
    params, arrays = emu.cache_params(c)
    params.update(mode=emu.MODE_ATTENTION, q_bf16=int(q_bf16), max_q=max_q, sm_scale=sm_scale)
    arrays.update(q=q, cu_q=np.asarray(cu_q, np.int32), lens=np.asarray(lens, np.int32),
                  signs=None if signs is None else np.asarray(signs, np.int8))
    total, lay = int(cu_q[-1]), c.layout
    r = emu.run(exe, tmp, params, arrays, {"out": (np.float32, (total, lay.num_q_heads, lay.head_dim)),
                                           "lse": (np.float32, (total, lay.num_q_heads))})
    return r["out"], r["lse"]


CASES = {
    # name: (workload overrides, chunk cap)
    "d64_g3_w16_k4v2": (dict(head_dim=64, num_q_heads=6, num_kv_heads=2, k_group=32, v_group=64, window=16), 70),
    "d128_g4_w0_whole_f32": (dict(window=0, in_dtype=wl.DT_F32), 10 ** 6),
    "d128_g5_allwindow": (dict(num_q_heads=10, num_kv_heads=2, window=1000), 30),
    "d128_g4_rot_w16": (dict(window=16, rotate_keys=True, outliers=("student_t", 2, 10.0, 3)), 70),
    "d64_g1_k8v8_w16": (dict(head_dim=64, num_q_heads=2, num_kv_heads=2, k_bits=8, v_bits=8, k_group=64,
                             v_group=64, window=16), 50),
    "d64_g2_k1v1_w8": (dict(head_dim=64, num_q_heads=4, num_kv_heads=2, k_bits=1, v_bits=1, k_group=32,
                            v_group=32, window=8), 65),
}

BASE = wl.Workload(name="prefill_emu", batch=3, num_q_heads=8, num_kv_heads=2, head_dim=128, seq_len=0,
                   k_bits=4, v_bits=2, k_group=32, v_group=128, window=16, ragged=(1, 200),
                   shuffle_pages=True, outliers=("random", 2, 10.0), seed=5)


@pytest.mark.parametrize("name", list(CASES))
def test_emulated_kernel_matches_oracle(emu_exe, tmp_path, name):
    over, cap = CASES[name]
    w = BASE.with_(**over)
    lens = wl.lengths(w)
    lens[-1] = max(int(lens[-1]), 130)             # at least three position tiles in one sequence
    signs = wl.rotation_signs(w) if w.rotate_keys else None
    pt = wl.page_table(w, np.maximum(0, lens - w.window))
    c = oracle.Cache(oracle.Layout.from_workload(w, signs), w.batch, pt, max(1, int((pt >= 0).sum())))
    kr, vr, _, _, cu, _ = wl.prefill(w, lens, with_f32=False)
    dt = oracle.IN_BF16 if w.in_dtype == wl.DT_BF16 else oracle.IN_F32
    c.append(kr, vr, dt, cu, np.zeros(w.batch, np.int32))
    n = np.minimum(lens, cap).astype(np.int32)
    cu_q = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    q, _ = wl.chunk_queries(w, int(cu_q[-1]))
    sc = 1 / np.sqrt(w.head_dim)
    ref_o, ref_l = c.prefill_attention(q, dt, cu_q, lens, sc)
    out, lse = _run(emu_exe, tmp_path, c, q, dt == oracle.IN_BF16, cu_q, lens, int(n.max()), sc, signs)
    np.testing.assert_allclose(out, ref_o, atol=ATOL, rtol=RTOL)
    np.testing.assert_allclose(lse, ref_l, atol=ATOL, rtol=RTOL)


def test_emulated_kernel_skips_empty_and_oversized_chunks(emu_exe, tmp_path):
    w = BASE.with_(window=8)
    lens = np.array([70, 0, 5], np.int32)
    pt = wl.page_table(w, np.maximum(0, lens - w.window))
    c = oracle.Cache(oracle.Layout.from_workload(w), w.batch, pt, max(1, int((pt >= 0).sum())))
    kr, vr, _, _, cu, _ = wl.prefill(w, lens, with_f32=False)
    c.append(kr, vr, oracle.IN_BF16, cu, np.zeros(w.batch, np.int32))
    # sequence 1 sends nothing; sequence 2 sends 7 queries for 5 positions (skipped, rows untouched)
    cu_q = np.array([0, 20, 20, 27], np.int32)
    q, _ = wl.chunk_queries(w, 27)
    out, lse = _run(emu_exe, tmp_path, c, q, True, cu_q, lens, 20, 0.125)
    ref_o, ref_l = c.prefill_attention(q[:20], oracle.IN_BF16, np.array([0, 20, 20, 20], np.int32),
                                       np.array([70, 0, 5], np.int32), 0.125)
    np.testing.assert_allclose(out[:20], ref_o, atol=ATOL, rtol=RTOL)
    np.testing.assert_allclose(lse[:20], ref_l, atol=ATOL, rtol=RTOL)
    assert np.all(out[20:] == 0) and np.all(lse[20:] == 0)


def _random_case(seed):
    """A random layout (d, GQA ratio, bits, grouping axis, groups, window,
    rotation, input type), ragged lengths including empty sequences, and a
    ragged chunk; seeded."""
    r = np.random.default_rng([seed, 77])
    d = int(r.choice([64, 128]))
    hkv, g = int(r.choice([1, 2])), int(r.choice([1, 2, 3, 4, 5, 8]))
    pc = bool(r.integers(0, 2))
    kg = int(r.choice([16, 32, 64])) if pc else int(r.choice([x for x in (16, 32, 64, 128) if x <= d]))
    w = wl.Workload(name="random", batch=int(r.integers(1, 4)), num_q_heads=hkv * g, num_kv_heads=hkv,
                    head_dim=d, seq_len=0, k_bits=int(r.choice([1, 2, 4, 8])), v_bits=int(r.choice([1, 2, 4, 8])),
                    k_group=kg, v_group=int(r.choice([x for x in (16, 32, 64, 128) if x <= d])),
                    window=int(r.choice([0, 1, 5, 16, 64, 200])), k_per_channel=pc,
                    rotate_keys=(not pc) and bool(r.integers(0, 4) == 0), ragged=(0, int(r.integers(1, 260))),
                    shuffle_pages=True, outliers=("random", 2, 10.0), seed=int(r.integers(0, 1 << 30)),
                    in_dtype=wl.DT_BF16 if r.integers(0, 3) else wl.DT_F32)
    cap = int(r.integers(1, 150))
    return w, r, cap


@pytest.mark.parametrize("seed", range(10))
def test_emulated_kernel_random_layouts(emu_exe, tmp_path, seed):
    w, r, cap = _random_case(seed)
    lens = wl.lengths(w)
    signs = wl.rotation_signs(w) if w.rotate_keys else None
    pt = wl.page_table(w, np.maximum(0, lens - w.window))
    c = oracle.Cache(oracle.Layout.from_workload(w, signs), w.batch, pt, max(1, int((pt >= 0).sum())))
    kr, vr, _, _, cu, _ = wl.prefill(w, lens, with_f32=False)
    dt = oracle.IN_BF16 if w.in_dtype == wl.DT_BF16 else oracle.IN_F32
    c.append(kr, vr, dt, cu, np.zeros(w.batch, np.int32))
    n = np.minimum(lens, r.integers(0, cap + 1, w.batch)).astype(np.int32)
    n[0] = min(int(lens[0]), max(1, int(n[0])))
    cu_q = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    if cu_q[-1] == 0:
        pytest.skip("every sequence of this draw is empty")
    q, _ = wl.chunk_queries(w, int(cu_q[-1]))
    sc = float(r.uniform(0.05, 0.2))
    ref_o, ref_l = c.prefill_attention(q, dt, cu_q, lens, sc)
    out, lse = _run(emu_exe, tmp_path, c, q, dt == oracle.IN_BF16, cu_q, lens, int(n.max()), sc, signs)
    np.testing.assert_allclose(out, ref_o, atol=ATOL, rtol=RTOL)
    np.testing.assert_allclose(lse, ref_l, atol=ATOL, rtol=RTOL)
