"""GPU parity of the chunked-prefill attention (kvq_prefill_attention)
against the oracle.

Each sequence first holds a context of L0 tokens (ragged, some empty); a
chunk of n new tokens (ragged, some zero, some longer than the window or
than one page) is appended to both caches through kvq_quantize_append /
the oracle, whose bytes must stay bit-identical; then the chunk's queries
attend causally over the cache.  Outputs and lse are compared with the
fp64 oracle within 1e-3 + 1e-3 * |ref|.
"""
import numpy as np
import pytest
import torch

import mixed_precision_quantized_kvq_b200 as kvq
import workloads as wl
from gpu_harness import Pair, check_close, in_code, torch_raw

pytestmark = pytest.mark.gpu


def small(**kw):
    base = dict(name="prefill", batch=4, num_q_heads=8, num_kv_heads=2, head_dim=128, seq_len=0,
                k_bits=4, v_bits=2, k_group=32, v_group=128, window=0, ragged=(1, 500),
                shuffle_pages=True, outliers=("random", 4, 10.0), seed=17)
    base.update(kw)
    return wl.Workload(**base)


def _chunk_rows(w, lens0, n):
    """Keys and values of positions [L0, L0 + n) of every sequence, stacked."""
    ks, vs = [], []
    for b in range(w.batch):
        if n[b] == 0:
            continue
        kr, vr, _, _ = wl.seq_kv(w, b, int(n[b]), start=int(lens0[b]))
        ks.append(kr)
        vs.append(vr)
    shape = (0, w.num_kv_heads, w.head_dim)
    rdt = np.uint16 if w.in_dtype == wl.DT_BF16 else np.float32
    return (np.concatenate(ks) if ks else np.empty(shape, rdt)), (np.concatenate(vs) if vs else np.empty(shape, rdt))


def run_chunk(w, lens0, n, want_lse=True):
    n = np.asarray(n, np.int32)
    pair = Pair(w, lens0, steps=int(n.max()))
    pair.prefill(with_f32=False)
    k, v = _chunk_rows(w, lens0, n)
    cu = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    pair.append(k, v, cu)
    pair.compare_cache()
    q, _ = wl.chunk_queries(w, int(cu[-1]), step=1)
    sc = 1.0 / np.sqrt(w.head_dim)
    out, lse = kvq.prefill_attention(pair.glay, pair.gcache, torch_raw(q), torch.from_numpy(cu).cuda(),
                                     pair.glens, int(n.max()), sc, want_lse=want_lse)
    torch.cuda.synchronize()
    ref, ref_lse = pair.ocache.prefill_attention(q, in_code(w), cu, pair.lens, sc)
    check_close(out.cpu().numpy(), ref, "out")
    if want_lse:
        check_close(lse.cpu().numpy(), ref_lse, "lse")
    return pair


@pytest.mark.parametrize("window", [0, 16, 128, 4096])
def test_chunk_after_context(window):
    w = small(window=window)
    lens0 = wl.lengths(w)
    lens0[1] = 0                                       # the chunk is the whole sequence
    n = [70, 130, 1, 0]                                # ragged, one empty chunk
    run_chunk(w, lens0, n)


@pytest.mark.parametrize("g", [1, 3, 4, 5, 8])
def test_gqa_ratios(g):
    w = small(num_q_heads=2 * g, window=64)
    lens0 = wl.lengths(w)
    run_chunk(w, lens0, [33, 64, 65, 7])


@pytest.mark.parametrize("kb,vb", [(4, 2), (2, 4), (8, 8), (1, 2), (4, 1)])
def test_bit_widths(kb, vb):
    w = small(k_bits=kb, v_bits=vb, window=32)
    run_chunk(w, wl.lengths(w), [50, 90, 3, 120])


def test_head_dim_64_and_fp32_inputs():
    w = small(head_dim=64, k_group=32, v_group=64, window=16, in_dtype=wl.DT_F32)
    run_chunk(w, wl.lengths(w), [40, 1, 77, 16], want_lse=False)


@pytest.mark.parametrize("window", [0, 48])
def test_key_rotation(window):
    w = small(rotate_keys=True, window=window, outliers=("student_t", 4, 10.0, 3))
    run_chunk(w, wl.lengths(w), [64, 100, 5, 31])


def test_whole_prompt_prefill_chunks():
    """Every sequence's chunk is its whole prompt (empty context)."""
    w = small(window=128)
    n = wl.lengths(w)
    run_chunk(w, np.zeros(w.batch, np.int32), n)


def test_skipped_sequences_leave_rows_untouched():
    """A chunk longer than its sequence is skipped; its rows keep their contents."""
    w = small(window=16, batch=2)
    pair = Pair(w, np.array([40, 10], np.int32))
    pair.prefill(with_f32=False)
    cu = torch.tensor([0, 5, 20], dtype=torch.int32, device="cuda")   # 15 queries for 10 positions
    q = torch_raw(wl.chunk_queries(w, 20)[0])
    out = torch.full((20, w.num_q_heads, w.head_dim), 3.0, device="cuda")
    lse = torch.full((20, w.num_q_heads), 3.0, device="cuda")
    kvq.kvq_prefill_attention(pair.glay, pair.gcache, q, cu, pair.glens, 15, 0.1, out, lse)
    torch.cuda.synchronize()
    assert torch.all(out[5:] == 3.0) and torch.all(lse[5:] == 3.0)
    ref, ref_lse = pair.ocache.prefill_attention(wl.chunk_queries(w, 20)[0][:5], in_code(w),
                                                 np.array([0, 5, 5], np.int32), pair.lens, 0.1)
    check_close(out[:5].cpu().numpy(), ref, "out")
    check_close(lse[:5].cpu().numpy(), ref_lse, "lse")


def test_argument_errors():
    w = small(window=16, batch=1)
    pair = Pair(w, np.array([10], np.int32))
    q = torch.zeros((1, w.num_q_heads, w.head_dim), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((1, w.num_q_heads, w.head_dim), device="cuda")
    cu = torch.tensor([0, 1], dtype=torch.int32, device="cuda")
    with pytest.raises(kvq.KVQError) as e:
        kvq.kvq_prefill_attention(pair.glay, pair.gcache, q, cu, pair.glens, -1, 0.1, out, None)
    assert e.value.status == kvq.KVQ_ERR_INVALID_ARG
    with pytest.raises(kvq.KVQError):
        kvq.kvq_prefill_attention(pair.glay, pair.gcache, q, cu, pair.glens, 1, float("nan"), out, None)
