"""kvq_decode_attention_static_scratch against kvq_decode_attention.

The static-scratch entry point runs the same plan and kernels as the
workspace entry point, with the split partials in the library's static
device array, so both must give bit-identical outputs.  Two calls in a row
on one stream also show that a call leaves nothing behind in the scratch
that changes the next one.  The file is named to be collected last, so the
static entry point runs both in a fresh process and after the other GPU
tests.
"""
import os
import re

import numpy as np
import pytest
import torch

import mixed_precision_quantized_kvq_b200 as kvq
import workloads as wl
from gpu_harness import Pair, torch_raw

pytestmark = pytest.mark.gpu

HEADER = os.path.join(os.path.dirname(__file__), "..", "include", "kvq.h")


def test_scratch_size_matches_header():
    text = open(HEADER).read()
    m = re.search(r"#define\s+KVQ_STATIC_SCRATCH_BYTES\s+\((\d+)u \* (\d+)u \* (\d+)u\)", text)
    assert m and int(m[1]) * int(m[2]) * int(m[3]) == kvq.KVQ_STATIC_SCRATCH_BYTES


@pytest.mark.parametrize("path", [kvq.DECODE_AUTO, kvq.DECODE_CUDA_CORES, kvq.DECODE_TCGEN05],
                         ids=["auto", "cuda_cores", "tcgen05"])
def test_two_calls_in_a_row_match_workspace_entry_point(path):
    w = wl.Workload(name="no_alloc", batch=6, num_q_heads=16, num_kv_heads=4, head_dim=128, seq_len=0,
                    k_bits=4, v_bits=2, k_group=32, v_group=128, window=40, ragged=(1, 2500),
                    shuffle_pages=True, outliers=("random", 4, 10.0), seed=21)
    lens = wl.lengths(w)
    lens[2] = 0
    kvq.kvq_set_decode_path(path)
    try:
        pair = Pair(w, lens)
        pair.prefill(with_f32=False)
        max_len = int(lens.max())
        sc = 1.0 / np.sqrt(w.head_dim)
        qs = [torch_raw(wl.query(w, step)[0]) for step in (0, 1)]
        shape_o, shape_l = (w.batch, w.num_q_heads, w.head_dim), (w.batch, w.num_q_heads)
        ws = kvq.workspace_for(pair.glay, w.batch, max_len, "cuda")
        assert ws.numel() * ws.element_size() <= kvq.KVQ_STATIC_SCRATCH_BYTES
        ref = []
        for q in qs:
            out = torch.empty(shape_o, dtype=torch.float32, device="cuda")
            lse = torch.empty(shape_l, dtype=torch.float32, device="cuda")
            kvq.kvq_decode_attention(pair.glay, pair.gcache, q, pair.glens, max_len, sc, out, lse, ws)
            ref.append((out, lse))
        got = [(torch.full(shape_o, 7.0, device="cuda"), torch.full(shape_l, 7.0, device="cuda")) for _ in qs]
        for q, (out, lse) in zip(qs, got):          # back to back on one stream
            kvq.kvq_decode_attention_static_scratch(pair.glay, pair.gcache, q, pair.glens, max_len, sc,
                                                    out, lse)
        torch.cuda.synchronize()
        for (ro, rl), (go, gl) in zip(ref, got):
            assert torch.equal(ro, go)
            assert torch.equal(rl, gl)
        assert not torch.equal(ref[0][0], ref[1][0])  # the two queries differ
    finally:
        kvq.kvq_set_decode_path(kvq.DECODE_AUTO)


def test_rejects_problem_larger_than_scratch():
    """On the two-phase tcgen05 path, whose split partials grow with the batch,
    batch 1024 x 32 query heads needs more than 16 MiB: refused on the host
    with KVQ_ERR_WORKSPACE, nothing launched, outputs untouched.  (The
    persistent kernel's partials are bounded by the SM count: about 1.3 MB.)"""
    lay = kvq.Layout(128, 32, 8, 4, 2, 32, 128, 64, 0)
    batch, max_len = 1024, 4096
    assert kvq.kvq_decode_workspace_bytes(lay, batch, max_len) < 2 * 1024 * 1024
    kvq.kvq_set_decode_path(kvq.DECODE_TCGEN05)
    try:
        _reject_large(lay, batch, max_len)
    finally:
        kvq.kvq_set_decode_path(kvq.DECODE_AUTO)


def _reject_large(lay, batch, max_len):
    assert kvq.kvq_decode_workspace_bytes(lay, batch, max_len) > kvq.KVQ_STATIC_SCRATCH_BYTES
    pt = torch.full((batch, 1), -1, dtype=torch.int32, device="cuda")
    cache = kvq.PagedCache.allocate(lay, pt, 1)
    q = torch.zeros((batch, 32, 128), dtype=torch.bfloat16, device="cuda")
    lens = torch.zeros(batch, dtype=torch.int32, device="cuda")
    out = torch.full((batch, 32, 128), 3.0, device="cuda")
    with pytest.raises(kvq.KVQError) as e:
        kvq.kvq_decode_attention_static_scratch(lay, cache, q, lens, max_len, 0.1, out, None)
    assert e.value.status == kvq.KVQ_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(out == 3.0)
