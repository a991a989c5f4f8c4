"""The C-ABI library loads, exports every entry point include/kvq.h declares,
and rejects bad arguments on the host with the documented status codes
(no GPU needed: every case here returns before any CUDA call)."""
import ctypes as C
import os
import re

import pytest

import mixed_precision_quantized_kvq_b200 as kvq
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    syms = set()
    for name in os.listdir(os.path.join(ROOT, "include")):
        if name.endswith(".h"):
            text = open(os.path.join(ROOT, "include", name)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            syms |= set(re.findall(r"\b(kvq_[a-z0-9_]+)\s*\(", text))
    return sorted(syms)


def test_header_declares_the_path():
    syms = declared_symbols()
    for s in ("kvq_quantize_append", "kvq_decode_attention", "kvq_dequantize"):
        assert s in syms


def test_library_exports_every_declared_symbol():
    lib = kvq.lib()
    missing = [s for s in declared_symbols() if not hasattr(lib, s)]
    assert not missing, missing


def test_binding_uses_abi_names():
    for s in declared_symbols():
        assert hasattr(kvq, s), s


def test_status_strings():
    for code in (0, -1, -2, -3, -4):
        assert kvq.kvq_status_string(code)
    assert kvq.kvq_status_string(7) == "unknown status"
    assert kvq.kvq_version() >= 100


def L(**kw):
    base = dict(head_dim=128, num_q_heads=32, num_kv_heads=8, k_bits=4, v_bits=2, k_group=32,
                v_group=128, window=128)
    base.update(kw)
    return kvq.Layout(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=96), kvq.KVQ_ERR_UNSUPPORTED),
    (dict(k_bits=3), kvq.KVQ_ERR_UNSUPPORTED),
    (dict(v_bits=16), kvq.KVQ_ERR_UNSUPPORTED),
    (dict(k_group=24), kvq.KVQ_ERR_UNSUPPORTED),
    (dict(head_dim=64, v_group=128), kvq.KVQ_ERR_UNSUPPORTED),
    (dict(num_q_heads=30), kvq.KVQ_ERR_UNSUPPORTED),
    (dict(num_q_heads=72), kvq.KVQ_ERR_UNSUPPORTED),          # GQA 9 > 8
    (dict(page_size=32), kvq.KVQ_ERR_UNSUPPORTED),
    (dict(window=-1), kvq.KVQ_ERR_INVALID_ARG),
    (dict(num_kv_heads=0), kvq.KVQ_ERR_INVALID_ARG),
    (dict(rotate_keys=True), kvq.KVQ_ERR_INVALID_ARG),        # no signs
])
def test_layout_rejected(kw, code):
    with pytest.raises(kvq.KVQError) as e:
        kvq.kvq_page_bytes(L(**kw))
    assert e.value.status == code


@pytest.mark.parametrize("kb,vb,kg,vg,d", [(4, 2, 32, 128, 128), (8, 8, 32, 128, 128),
                                           (1, 2, 32, 128, 128), (4, 2, 32, 64, 64),
                                           (2, 4, 16, 64, 64)])
def test_page_bytes_agree_with_oracle(kb, vb, kg, vg, d):
    lay = L(head_dim=d, k_bits=kb, v_bits=vb, k_group=kg, v_group=vg)
    got = kvq.kvq_page_bytes(lay)
    want = oracle.page_bytes(oracle.Layout(d, 32, 8, kb, vb, kg, vg, 64, 128))
    assert got == want
    assert kvq.kvq_window_bytes(lay, 16) == 16 * 8 * 128 * d * 2


def _fake_cache(batch=2, window=True):
    # host buffers stand in for device memory; nothing is launched in these cases
    bufs = [C.create_string_buffer(4096) for _ in range(7)]
    addr = lambda b: (C.addressof(b) + 15) & ~15
    c = kvq.kvq_cache(addr(bufs[0]), addr(bufs[1]), addr(bufs[2]), addr(bufs[3]),
                      addr(bufs[4]) if window else None, addr(bufs[5]) if window else None,
                      addr(bufs[6]), batch, 4, 8)
    return c, bufs


def test_entry_points_reject_bad_arguments_on_host():
    lib = kvq.lib()
    lay = L()
    c, keep = _fake_cache()
    buf = C.create_string_buffer(1024)
    p = C.c_void_p((C.addressof(buf) + 255) & ~255)
    null = None
    # append
    assert lib.kvq_quantize_append(None, C.byref(c), p, p, 1, p, p, 4, null) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_quantize_append(C.byref(lay.c()), None, p, p, 1, p, p, 4, null) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_quantize_append(C.byref(lay.c()), C.byref(c), p, p, 7, p, p, 4, null) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_quantize_append(C.byref(lay.c()), C.byref(c), None, p, 1, p, p, 4, null) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_quantize_append(C.byref(lay.c()), C.byref(c), p, p, 1, None, p, 4, null) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_quantize_append(C.byref(lay.c()), C.byref(c), p, p, 1, p, p, -1, null) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_quantize_append(C.byref(lay.c()), C.byref(c), p, p, 1, p, p, 0, null) == kvq.KVQ_OK
    bad = L(k_bits=3)
    assert lib.kvq_quantize_append(C.byref(bad.c()), C.byref(c), p, p, 1, p, p, 4, null) == kvq.KVQ_ERR_UNSUPPORTED
    # window buffers are required when the layout has a window
    c2, keep2 = _fake_cache(window=False)
    assert lib.kvq_quantize_append(C.byref(lay.c()), C.byref(c2), p, p, 1, p, p, 4, null) == kvq.KVQ_ERR_INVALID_ARG
    # misaligned buffer
    c3, keep3 = _fake_cache()
    c3.k_codes = c3.k_codes + 4
    assert lib.kvq_quantize_append(C.byref(lay.c()), C.byref(c3), p, p, 1, p, p, 4, null) == kvq.KVQ_ERR_INVALID_ARG
    # decode: missing / short / misaligned workspace
    args = lambda ws, n: (C.byref(lay.c()), C.byref(c), p, 1, p, 4096, C.c_float(0.088), p, None, ws, n, null)
    assert lib.kvq_decode_attention(*args(None, 0)) == kvq.KVQ_ERR_WORKSPACE
    assert lib.kvq_decode_attention(*args(p, 16)) == kvq.KVQ_ERR_WORKSPACE
    assert lib.kvq_decode_attention(C.byref(lay.c()), C.byref(c), p, 5, p, 4096, C.c_float(0.1), p, None, p,
                                    1 << 30, null) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_decode_attention(C.byref(lay.c()), C.byref(c), p, 1, p, 4096, C.c_float(float("nan")), p,
                                    None, p, 1 << 30, null) == kvq.KVQ_ERR_INVALID_ARG
    # dequantize / rotate
    assert lib.kvq_dequantize(C.byref(lay.c()), C.byref(c), p, 10, None, p, null) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_dequantize(C.byref(lay.c()), C.byref(c), p, 0, p, p, null) == kvq.KVQ_OK
    assert lib.kvq_rotate_keys(C.byref(lay.c()), p, 1, 4, p, null) == kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_rotate_keys(None, p, 1, 4, p, null) == kvq.KVQ_ERR_INVALID_ARG


def test_workspace_size_monotone():
    lay = L()
    a = kvq.kvq_decode_workspace_bytes(lay, 16, 4096)
    assert a > 0
    assert kvq.kvq_decode_workspace_bytes(lay, 0, 4096) >= 0
    assert kvq.kvq_decode_workspace_bytes(L(k_bits=3), 16, 4096) == 0
    assert kvq.kvq_decode_workspace_bytes(lay, 16, -1) == 0


@pytest.mark.parametrize("kb,vb,kg,vg,d,w", [(4, 2, 64, 128, 128, 128), (4, 2, 32, 128, 128, 0),
                                             (2, 4, 16, 64, 64, 8), (1, 1, 16, 32, 64, 3)])
def test_per_channel_sizes_agree_with_oracle(kb, vb, kg, vg, d, w):
    """Key groups along positions: page bytes as the oracle's layout, a ring
    of window + k_group - 1 slots, no decode workspace; head_dim 128 decodes
    with the per-channel kernel, head_dim 64 on CUDA cores."""
    lay = L(head_dim=d, k_bits=kb, v_bits=vb, k_group=kg, v_group=vg, window=w, k_per_channel=True)
    olay = oracle.Layout(d, 32, 8, kb, vb, kg, vg, 64, w, k_per_channel=True)
    assert kvq.kvq_page_bytes(lay) == oracle.page_bytes(olay)
    assert kvq.kvq_window_bytes(lay, 16) == 16 * 8 * (w + kg - 1) * d * 2 == 16 * 8 * olay.ring_slots * d * 2
    assert kvq.kvq_decode_workspace_bytes(lay, 16, 4096) == 0
    assert kvq.kvq_get_decode_path(lay) == (kvq.DECODE_PER_CHANNEL if d == 128 else kvq.DECODE_CUDA_CORES)


@pytest.mark.parametrize("kw,code", [
    (dict(k_group=128), kvq.KVQ_ERR_UNSUPPORTED),             # a group must fit in a 64-position page
    (dict(k_group=48), kvq.KVQ_ERR_UNSUPPORTED),
    (dict(rotate_keys=True), kvq.KVQ_ERR_UNSUPPORTED),        # checked before the missing signs
])
def test_per_channel_layout_rejected(kw, code):
    with pytest.raises(kvq.KVQError) as e:
        kvq.kvq_page_bytes(L(k_per_channel=True, **kw))
    assert e.value.status == code


def test_per_channel_ring_required_without_window():
    """With key groups along positions the ring exists even at window 0."""
    lib = kvq.lib()
    lay = L(window=0, k_per_channel=True)
    c, keep = _fake_cache(window=False)
    buf = C.create_string_buffer(1024)
    p = C.c_void_p((C.addressof(buf) + 255) & ~255)
    assert lib.kvq_quantize_append(C.byref(lay.c()), C.byref(c), p, p, 1, p, p, 4, None) == kvq.KVQ_ERR_INVALID_ARG


def test_per_channel_split_workspace_rule():
    """Key groups along positions: the decode splits pairs between CTAs only
    when the pairs leave SMs idle (148 SMs without a device) and the sequences
    hold eight 64-position tiles per CTA; the workspace then holds a part of
    8 heads x 132 floats per (pair, split), 256-byte aligned, and a ticket per
    pair."""
    lay = L(k_group=64, v_group=64, window=0, k_per_channel=True)
    assert kvq.kvq_decode_workspace_bytes(lay, 16, 4096) == 0        # 128 pairs: one CTA each
    assert kvq.kvq_decode_workspace_bytes(lay, 8, 511) == 0          # too short to split
    pairs = 8 * 8                                                    # B8: 64 pairs, two CTAs each
    part = (pairs * 2 * 8 * 132 * 4 + 255) // 256 * 256
    assert kvq.kvq_decode_workspace_bytes(lay, 8, 16384) == part + pairs * 4
    pairs = 1 * 8                                                    # B1: 8 pairs, eight CTAs each
    part = (pairs * 8 * 8 * 132 * 4 + 255) // 256 * 256
    assert kvq.kvq_decode_workspace_bytes(lay, 1, 16384) == part + pairs * 4
    assert kvq.kvq_decode_workspace_bytes(L(head_dim=64, k_group=64, v_group=64, window=0, k_per_channel=True),
                                          1, 16384) == 0             # head_dim 64: the chunked-prefill path
