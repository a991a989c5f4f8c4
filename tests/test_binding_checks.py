"""The Python binding checks buffers before it calls the library: a tensor
of the wrong dtype, size or device raises ValueError instead of reaching a
kernel that would read or write past its end."""
import numpy as np
import pytest
import torch

import mixed_precision_quantized_kvq_b200 as kvq


def _layout():
    return kvq.Layout(128, 32, 8, 4, 2, 32, 128, 64, 16)


def _cache(device="cpu", batch=2):
    lay = _layout()
    pt = torch.arange(batch * 4, dtype=torch.int32, device=device).reshape(batch, 4)
    z = lambda: torch.zeros(64, dtype=torch.uint8, device=device)
    return lay, kvq.PagedCache(z(), z(), z(), z(), z(), z(), pt, batch * 4)


def test_host_tensors_are_rejected():
    """No CUDA device needed: host tensors fail the check before any call."""
    lay, c = _cache()
    B = c.batch
    q = torch.zeros((B, 32, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        kvq.kvq_decode_attention(lay, c, q, torch.zeros(B, dtype=torch.int32), 10, 0.1,
                                 torch.zeros((B, 32, 128)), None, torch.zeros(256, dtype=torch.uint8))
    with pytest.raises(ValueError, match="CUDA tensor"):
        kvq.kvq_quantize_append(lay, c, torch.zeros((B, 8, 128)), torch.zeros((B, 8, 128)),
                                torch.zeros(B + 1, dtype=torch.int32), torch.zeros(B, dtype=torch.int32), 1)
    with pytest.raises(ValueError, match="CUDA tensor"):
        kvq.kvq_dequantize(lay, c, torch.zeros(B, dtype=torch.int32), 4, torch.zeros(1), torch.zeros(1))


def test_append_decode_checks_both_calls_arguments():
    """kvq_append_decode checks the append's and the decode's buffers."""
    lay, c = _cache()
    B = c.batch
    kv = torch.zeros((B, 8, 128))
    args = dict(cu_new=torch.zeros(B + 1, dtype=torch.int32), lens_old=torch.zeros(B, dtype=torch.int32),
                max_new=1, q=torch.zeros((B, 32, 128), dtype=torch.bfloat16),
                lens=torch.ones(B, dtype=torch.int32), max_len=1, sm_scale=0.1, out=torch.zeros((B, 32, 128)),
                lse=None, workspace=torch.zeros(256, dtype=torch.uint8))
    with pytest.raises(ValueError, match="CUDA tensor"):
        kvq.kvq_append_decode(lay, c, kv, kv, **args)
    with pytest.raises(ValueError, match="share a dtype"):
        kvq.kvq_append_decode(lay, c, kv, kv.to(torch.bfloat16), **args)
    with pytest.raises(ValueError):
        kvq.kvq_append_decode(lay, c, kv, kv, **dict(args, lens_old=torch.zeros(B + 1, dtype=torch.int32)))


def test_mismatched_key_value_dtypes_are_rejected():
    lay, c = _cache()
    with pytest.raises(ValueError, match="share a dtype"):
        kvq.kvq_quantize_append(lay, c, torch.zeros((2, 8, 128)), torch.zeros((2, 8, 128), dtype=torch.bfloat16),
                                torch.zeros(3, dtype=torch.int32), torch.zeros(2, dtype=torch.int32), 1)


@pytest.mark.gpu
def test_wrong_dtype_and_size_are_rejected_on_the_device():
    lay, c = _cache("cuda")
    B = c.batch
    q = torch.zeros((B, 32, 128), dtype=torch.bfloat16, device="cuda")
    lens = torch.full((B,), 8, dtype=torch.int32, device="cuda")
    out = torch.zeros((B, 32, 128), device="cuda")
    ws = kvq.workspace_for(lay, B, 8, "cuda")
    bad_out = [torch.zeros((B, 32, 128), dtype=torch.bfloat16, device="cuda"),   # bf16 output
               torch.zeros((B, 32, 127), device="cuda")]                        # too small
    for o in bad_out:
        with pytest.raises(ValueError):
            kvq.kvq_decode_attention(lay, c, q, lens, 8, 0.1, o, None, ws)
    with pytest.raises(ValueError, match="dtype"):
        kvq.kvq_decode_attention(lay, c, q, lens.to(torch.int64), 8, 0.1, out, None, ws)
    with pytest.raises(ValueError, match="elements"):
        kvq.kvq_decode_attention(lay, c, q, lens, 8, 0.1, out, torch.zeros(B, device="cuda"), ws)
    with pytest.raises(ValueError, match="elements"):
        kvq.kvq_decode_attention(lay, c, q, lens, 8, 0.1, out, None, ws[:16])
    with pytest.raises(ValueError, match="elements"):
        kvq.kvq_quantize_append(lay, c, torch.zeros((B, 8, 128), device="cuda"), torch.zeros((B, 8, 128), device="cuda"),
                                torch.zeros(B, dtype=torch.int32, device="cuda"), lens, 1)
