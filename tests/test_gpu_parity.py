"""GPU parity against the CPU oracle on small and medium cases (several
pages, ragged tails, empty sequences, all bit widths, GQA 1/4/5/8, windows,
rotation, incremental appends).  Codes, metadata and window bytes must be
bit-identical; attention outputs within |err| <= 1e-3 + 1e-3*|ref| of the
fp64 oracle on the same reconstructed cache."""
import numpy as np
import pytest
import torch

import mixed_precision_quantized_kvq_b200 as kvq
import oracle
import workloads as wl
from gpu_harness import Pair, check_close, torch_raw

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, params=[kvq.DECODE_AUTO, kvq.DECODE_CUDA_CORES, kvq.DECODE_TCGEN05],
                ids=["auto", "cuda_cores", "tcgen05"])
def decode_path(request):
    """Every case runs on the automatic choice (the persistent tensor-core
    kernel where the layout allows), on the CUDA-core kernel and on the
    two-phase tcgen05 kernel."""
    kvq.kvq_set_decode_path(request.param)
    yield request.param
    kvq.kvq_set_decode_path(kvq.DECODE_AUTO)


def test_tensor_core_path_selected_for_k4v2_layout(decode_path):
    lay = kvq.Layout(128, 32, 8, 4, 2, 32, 128, 64, 128)
    want = {kvq.DECODE_AUTO: kvq.DECODE_TENSOR_CORES, kvq.DECODE_CUDA_CORES: kvq.DECODE_CUDA_CORES,
            kvq.DECODE_TCGEN05: kvq.DECODE_TCGEN05}[decode_path]
    assert kvq.kvq_get_decode_path(lay) == want
    assert kvq.kvq_get_decode_path(kvq.Layout(64, 4, 4, 4, 2, 32, 64, 64, 0)) == kvq.DECODE_CUDA_CORES


def small(**kw):
    base = dict(name="small", batch=4, num_q_heads=8, num_kv_heads=2, head_dim=128, seq_len=0,
                k_bits=4, v_bits=2, k_group=32, v_group=128, window=0, ragged=(1, 700),
                shuffle_pages=True, outliers=("random", 4, 10.0), seed=7)
    base.update(kw)
    return wl.Workload(**base)


def run_prefill_and_decode(w, lens=None):
    lens = wl.lengths(w) if lens is None else np.asarray(lens, np.int32)
    pair = Pair(w, lens)
    pair.prefill()
    pair.compare_cache()
    pair.check_decode()
    return pair


def test_tiny_workload():
    """The tiny K4V2 workload (fp32 inputs, head_dim 64, 256 tokens)."""
    w = wl.TINY
    pair = run_prefill_and_decode(w)
    k, v = pair.dequantize()
    ko, vo = pair.ocache.dequantize(pair.lens, int(pair.lens.max()))
    np.testing.assert_array_equal(k, ko)
    np.testing.assert_array_equal(v, vo)


@pytest.mark.parametrize("kb,vb", [(8, 8), (4, 4), (4, 2), (2, 4), (2, 2), (1, 2), (1, 1), (8, 1)])
def test_bit_widths(kb, vb):
    run_prefill_and_decode(small(k_bits=kb, v_bits=vb))


@pytest.mark.parametrize("d,kg,vg", [(128, 16, 16), (128, 32, 64), (128, 64, 128), (128, 128, 32),
                                     (64, 32, 64), (64, 16, 32), (64, 64, 16)])
def test_groups_and_head_dims(d, kg, vg):
    run_prefill_and_decode(small(head_dim=d, k_group=kg, v_group=vg))


@pytest.mark.parametrize("hq,hkv", [(2, 2), (8, 2), (10, 2), (16, 2), (6, 6)])
def test_gqa(hq, hkv):
    run_prefill_and_decode(small(num_q_heads=hq, num_kv_heads=hkv))


@pytest.mark.parametrize("window", [1, 64, 100, 5000])
def test_windows(window):
    lens = wl.lengths(small())
    lens[0] = 0
    lens[1] = 3
    run_prefill_and_decode(small(window=window), lens)


def test_fp32_inputs_with_window():
    run_prefill_and_decode(small(in_dtype=wl.DT_F32, window=40, head_dim=64, k_group=32, v_group=64))


@pytest.mark.parametrize("d,vg", [(64, 64), (128, 128)])
def test_rotation(d, vg):
    w = small(rotate_keys=True, head_dim=d, v_group=vg, outliers=("student_t", 4, 10.0, 3.0))
    lens = wl.lengths(w)
    kr, vr, kf, vf, cu, _ = wl.prefill(w, lens)
    pair = Pair(w, lens)
    # rotated keys, as the library computes them before quantizing
    kt = torch_raw(kr)
    rot = torch.empty(kt.shape, dtype=torch.float32, device="cuda")
    kvq.kvq_rotate_keys(pair.glay, kt, rot)
    rot = rot.cpu().numpy()
    # the fast transform agrees with the oracle's dense fp64 rotation to round-off
    ref = oracle.rotate(kf.reshape(-1, d)[:4000], pair.signs).reshape(-1, d)
    scale = np.abs(kf.reshape(-1, d)[:4000]).max(axis=1, keepdims=True)
    assert np.all(np.abs(rot.reshape(-1, d)[:4000] - ref) <= 2.0 ** -20 * scale * np.sqrt(d))
    # codes: the oracle quantizes the library's rotated keys
    olay = oracle.Layout.from_workload(w.with_(rotate_keys=False))
    pair.ocache = oracle.Cache(olay, w.batch, pair.pt, pair.num_pages)
    pair.lens[:] = 0
    pair.glens.zero_()
    pair.append(kr, vr, cu, oracle_k=np.ascontiguousarray(rot), oracle_dtype=oracle.IN_F32)
    pair.compare_cache()
    # attention: quantized keys are in the rotated domain, the query is rotated
    pair.ocache.layout = pair.olay
    pair.ocache._signs = np.ascontiguousarray(pair.signs)
    pair.check_decode()


def test_incremental_appends_and_decode_steps():
    w = small(window=48, ragged=(1, 300))
    final = wl.lengths(w)
    steps = 5
    pair = Pair(w, final, steps=steps + 200)
    kr, vr, kf, vf, cu, _ = wl.prefill(w, final)
    pair.lens[:] = 0
    pair.glens.zero_()
    r = np.random.default_rng(3)
    done = np.zeros(w.batch, np.int32)
    while np.any(done < final):                       # chunked prefill, chunks of 0..90
        n = np.minimum(r.integers(0, 90, w.batch), final - done).astype(np.int32)
        ks = np.concatenate([kr[cu[b] + done[b]: cu[b] + done[b] + n[b]] for b in range(w.batch)])
        vs = np.concatenate([vr[cu[b] + done[b]: cu[b] + done[b] + n[b]] for b in range(w.batch)])
        cun = np.zeros(w.batch + 1, np.int32)
        cun[1:] = np.cumsum(n)
        pair.append(ks, vs, cun)
        done += n
    pair.compare_cache()
    for s in range(steps):                            # decode: one token per sequence
        k1, v1, _, _ = wl.new_tokens(w, s)
        pair.append(k1, v1, np.arange(w.batch + 1, dtype=np.int32))
        pair.compare_cache()
        pair.check_decode(step=s)


def test_empty_and_single_token_sequences():
    w = small(window=0)
    run_prefill_and_decode(w, np.array([0, 1, 64, 65], np.int32))
    run_prefill_and_decode(small(window=16), np.array([0, 0, 0, 0], np.int32))


def test_lse_and_output_of_empty_sequence():
    w = small()
    pair = Pair(w, np.array([0, 5, 0, 129], np.int32))
    pair.prefill()
    _, out, lse = pair.decode()
    assert np.all(out[0] == 0) and np.all(np.isneginf(lse[0]))
    assert np.all(out[2] == 0) and np.all(np.isneginf(lse[2]))


def test_max_len_larger_than_lengths():
    w = small()
    pair = Pair(w, wl.lengths(w))
    pair.prefill()
    qr, out, lse = pair.decode(max_len=int(pair.lens.max()) + 1000)
    ref, _ = pair.oracle_decode(qr)
    check_close(out, ref)


@pytest.mark.parametrize("window", [48, 200])
def test_rotation_with_window(window):
    """Rotated keys in pages, unrotated keys in the bf16 window: each scored
    against the matching query."""
    w = small(rotate_keys=True, window=window, ragged=(1, 900),
              outliers=("student_t", 4, 10.0, 3.0))
    lens = wl.lengths(w)
    kr, vr, kf, vf, cu, _ = wl.prefill(w, lens)
    pair = Pair(w, lens)
    kt = torch_raw(kr)
    rot = torch.empty(kt.shape, dtype=torch.float32, device="cuda")
    kvq.kvq_rotate_keys(pair.glay, kt, rot)
    rot = rot.cpu().numpy()
    # oracle rows: rotated keys where the position ends up quantized, raw keys in the window
    ok_rows = kf.astype(np.float32).copy()
    for b in range(w.batch):
        nq = max(0, int(lens[b]) - window)
        ok_rows[cu[b]:cu[b] + nq] = rot[cu[b]:cu[b] + nq]
    olay = oracle.Layout.from_workload(w.with_(rotate_keys=False))
    pair.ocache = oracle.Cache(olay, w.batch, pair.pt, pair.num_pages)
    pair.lens[:] = 0
    pair.glens.zero_()
    pair.append(kr, vr, cu, oracle_k=np.ascontiguousarray(ok_rows), oracle_dtype=oracle.IN_F32)
    # the oracle's window holds fp32 rows rounded to bf16 (exact: they came from bf16)
    pair.compare_cache()
    pair.ocache.layout = pair.olay
    pair.ocache._signs = np.ascontiguousarray(pair.signs)
    pair.check_decode()


@pytest.mark.parametrize("window,n,in_dtype", [(0, 3, wl.DT_BF16), (8, 8, wl.DT_BF16), (64, 2, wl.DT_BF16),
                                               (5, 5, wl.DT_F32), (100, 1, wl.DT_BF16), (3, 1, wl.DT_F32)])
def test_small_appends_after_prefill(window, n, in_dtype):
    """Appends of n <= 8 tokens per sequence, at most the window, take the
    single-launch append path: ring slots are read, refilled with the new
    tokens and the old rows quantized in one pass; value words are merged
    bit-field by bit-field.  Cache bytes stay bit-identical to the oracle."""
    w = small(window=window, ragged=(1, 300), in_dtype=in_dtype)
    lens = wl.lengths(w)
    lens[0] = 0                                        # an empty sequence that starts filling
    lens[1] = min(window, 3)                           # a ring that is not yet full
    steps = 4
    pair = Pair(w, lens, steps=steps * n + 8)
    pair.prefill()
    for s in range(steps):
        toks = [wl.new_tokens(w, 100 + s * n + i) for i in range(n)]
        k = np.stack([t[0] for t in toks], axis=1).reshape(w.batch * n, w.num_kv_heads, w.head_dim)
        v = np.stack([t[1] for t in toks], axis=1).reshape(w.batch * n, w.num_kv_heads, w.head_dim)
        pair.append(k, v, np.arange(w.batch + 1, dtype=np.int32) * n)
        pair.compare_cache()
        pair.check_decode(step=s)
