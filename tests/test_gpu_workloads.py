"""GPU parity on the five workloads at full size, in the launch
configuration the benchmark times: codes, metadata and window bytes
bit-identical to the oracle over the whole cache; attention outputs within
1e-3 + 1e-3*|ref| of the fp64 oracle on the same reconstructed cache."""
import numpy as np
import pytest
import torch

import mixed_precision_quantized_kvq_b200 as kvq
import oracle
import workloads as wl
from gpu_harness import Pair, torch_raw

pytestmark = pytest.mark.gpu


def test_llama8b_layer_full():
    """B16, 32/8 heads, d128, 4096 cached tokens, K4 g32 / V2 g128, W128."""
    w = wl.LLAMA8B
    pair = Pair(w, wl.lengths(w), steps=2)
    pair.prefill(with_f32=False)
    pair.compare_cache()
    pair.check_decode(step=0)
    for s in range(2):                      # decode steps: append one token, attend
        k1, v1, _, _ = wl.new_tokens(w, s)
        pair.append(k1, v1, np.arange(w.batch + 1, dtype=np.int32))
        pair.check_decode(step=s + 1)
    pair.compare_cache()


@pytest.mark.parametrize("kb,vb", wl.SWEEP_BITS)
def test_bit_allocation_sweep_full(kb, vb):
    """B8, 32/8 heads, d128, 16384 tokens at K8V8 ... K1V2."""
    w = wl.SWEEP.with_(k_bits=kb, v_bits=vb)
    pair = Pair(w, wl.lengths(w))
    pair.prefill(with_f32=False)
    pair.compare_cache()
    pair.check_decode(step=0)


def test_ragged_paged_full():
    """64 sequences, L ~ U[512, 16384], shuffled pages, GQA 5, W64: prefill,
    then 32 decode steps that each append one token per sequence."""
    w = wl.RAGGED
    lens = wl.lengths(w)
    pair = Pair(w, lens, steps=w.decode_steps)
    pair.prefill(with_f32=False)
    pair.compare_cache()
    for s in range(w.decode_steps):
        k1, v1, _, _ = wl.new_tokens(w, s)
        pair.append(k1, v1, np.arange(w.batch + 1, dtype=np.int32))
        if s in (0, w.decode_steps - 1):
            pair.check_decode(step=s)
    pair.compare_cache()


def test_rotation_full():
    """B32, 32/8 heads, d128, 8192 tokens, K4V2, keys rotated."""
    w = wl.ROTATION
    lens = wl.lengths(w)
    pair = Pair(w, lens)
    kr, vr, _, _, cu, _ = wl.prefill(w, lens, with_f32=False)
    rot = torch.empty(kr.shape, dtype=torch.float32, device="cuda")
    kvq.kvq_rotate_keys(pair.glay, torch_raw(kr), rot)
    rot = rot.cpu().numpy()
    olay = oracle.Layout.from_workload(w.with_(rotate_keys=False))
    pair.ocache = oracle.Cache(olay, w.batch, pair.pt, pair.num_pages)
    pair.lens[:] = 0
    pair.glens.zero_()
    pair.append(kr, vr, cu, oracle_k=rot, oracle_dtype=oracle.IN_F32)
    pair.compare_cache()
    pair.ocache.layout = pair.olay
    pair.ocache._signs = np.ascontiguousarray(pair.signs)
    pair.check_decode(step=0)
