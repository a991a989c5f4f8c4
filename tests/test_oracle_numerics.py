"""Pins of the oracle's number-format helpers against independent references.

* binary16 conversion in three rounding directions: every finite binary16
  value, the boundaries between neighbours, overflow and subnormals; round to
  nearest is compared with numpy's float16 cast, directed rounding with the
  bracketing neighbours numpy enumerates.
* bfloat16 round-to-nearest against torch's bfloat16 cast.
* fp32 subtraction / division rounded up against exact rational arithmetic,
  and rounded to nearest against numpy's fp32 arithmetic.
"""
import math
import random
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

F16_POS = np.arange(0x0000, 0x7C00, dtype=np.uint16)        # +0 .. 65504
F16_POS_VAL = F16_POS.view(np.float16).astype(np.float32)


def test_every_finite_f16_value_is_fixed_point():
    for sign in (0, 0x8000):
        bits = (F16_POS | np.uint16(sign)).astype(np.uint16)
        vals = bits.view(np.float16).astype(np.float32)
        for mode in (oracle.RN, oracle.RD, oracle.RU):
            got = oracle.f32_to_f16(vals, mode)
            np.testing.assert_array_equal(got, bits)


def _between_points():
    lo = F16_POS_VAL[:-1].astype(np.float32)
    hi = F16_POS_VAL[1:].astype(np.float32)
    mid = ((lo.astype(np.float64) + hi.astype(np.float64)) / 2).astype(np.float32)
    assert np.all(mid.astype(np.float64) == (lo.astype(np.float64) + hi.astype(np.float64)) / 2)
    pts = [np.nextafter(lo, np.float32(np.inf)), np.nextafter(mid, np.float32(-np.inf)), mid,
           np.nextafter(mid, np.float32(np.inf)), np.nextafter(hi, np.float32(-np.inf))]
    return lo, hi, pts


def test_f16_directed_brackets_and_adjacency():
    lo, hi, pts = _between_points()
    lo_bits, hi_bits = F16_POS[:-1], F16_POS[1:]
    for x in pts:
        np.testing.assert_array_equal(oracle.f32_to_f16(x, oracle.RD), lo_bits)
        np.testing.assert_array_equal(oracle.f32_to_f16(x, oracle.RU), hi_bits)
        # mirror image for negative inputs
        np.testing.assert_array_equal(oracle.f32_to_f16(-x, oracle.RU), lo_bits | 0x8000)
        np.testing.assert_array_equal(oracle.f32_to_f16(-x, oracle.RD), hi_bits | 0x8000)


def test_f16_nearest_matches_numpy_cast():
    _, _, pts = _between_points()
    r = np.random.default_rng(11)
    rand = [r.standard_normal(400_000).astype(np.float32) * s for s in (1e-6, 1e-3, 1.0, 1e3, 3e4)]
    for x in pts + rand:
        for sx in (x, -x):
            with np.errstate(over="ignore"):
                want = sx.astype(np.float16).view(np.uint16)
            np.testing.assert_array_equal(oracle.f32_to_f16(sx, oracle.RN), want)


@pytest.mark.parametrize("x,mode,bits", [
    (65504.5, oracle.RU, 0x7C00), (65504.5, oracle.RD, 0x7BFF), (1e6, oracle.RD, 0x7BFF),
    (65519.0, oracle.RN, 0x7BFF), (65520.0, oracle.RN, 0x7C00), (-1e6, oracle.RD, 0xFC00),
    (-1e6, oracle.RU, 0xFBFF), (1e-10, oracle.RU, 0x0001), (1e-10, oracle.RD, 0x0000),
    (-1e-10, oracle.RD, 0x8001), (-1e-10, oracle.RU, 0x8000), (2.0 ** -25, oracle.RN, 0x0000),
    (2.0 ** -25 * 1.5, oracle.RN, 0x0001), (3 * 2.0 ** -25, oracle.RN, 0x0002),
])
def test_f16_edges(x, mode, bits):
    assert int(oracle.f32_to_f16(np.float32(x), mode)[0]) == bits


def test_f16_decode_matches_numpy():
    allbits = np.arange(0, 0x10000, dtype=np.uint32).astype(np.uint16)
    finite = allbits[(allbits & 0x7C00) != 0x7C00]
    sample = finite[:: 7]
    want = sample.view(np.float16).astype(np.float32)
    got = oracle.f16_to_f32(sample)
    np.testing.assert_array_equal(got.view(np.uint32), want.view(np.uint32))


def test_bf16_nearest_matches_torch():
    r = np.random.default_rng(12)
    x = np.concatenate([r.standard_normal(300_000).astype(np.float32) * s
                        for s in (1e-30, 1e-3, 1.0, 1e4, 1e30)])
    # exact ties: low 16 bits == 0x8000
    ties = (r.integers(0, 2 ** 31, 5000, dtype=np.uint32) & np.uint32(0xFFFF0000)) | np.uint32(0x8000)
    x = np.concatenate([x, ties.view(np.float32)])
    x = x[np.isfinite(x)]
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(oracle.f32_to_bf16(x, oracle.RN), want)


def _next_down(f: float) -> float:
    return float(np.nextafter(np.float32(f), np.float32(-np.inf)))


def _pairs(n, seed):
    r = random.Random(seed)
    out = []
    specials = [0.0, -0.0, 1.0, -1.0, 3.0, 15.0, 255.0, 1e-38, 1e-45, 65504.0, 7.0, 1.0 / 3]
    for _ in range(n):
        kind = r.random()
        if kind < 0.2:
            a, b = r.choice(specials), r.choice(specials)
        else:
            a = r.uniform(-1, 1) * 10 ** r.uniform(-8, 6)
            b = r.uniform(-1, 1) * 10 ** r.uniform(-8, 6)
        out.append((float(np.float32(a)), float(np.float32(b))))
    return out


def test_directed_sub_div_against_exact_rationals():
    pairs = _pairs(6000, 13)
    a = np.array([p[0] for p in pairs], np.float32)
    b = np.array([p[1] for p in pairs], np.float32)
    sub = oracle.fp_op(a, b, "sub", up=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        bb = np.where(b == 0, np.float32(3.0), b)
    div = oracle.fp_op(a, bb, "div", up=True)
    for i in range(len(pairs)):
        for got, exact in ((sub[i], Fraction(float(a[i])) - Fraction(float(b[i]))),
                           (div[i], Fraction(float(a[i])) / Fraction(float(bb[i])))):
            g = float(got)
            if abs(exact) >= Fraction(2) ** 128:           # beyond fp32: overflow
                want = math.inf if exact > 0 else -float(np.finfo(np.float32).max)
                assert g == want
                continue
            assert math.isfinite(g)
            assert Fraction(g) >= exact                      # rounded up
            if Fraction(g) != exact:                         # and by the least amount
                assert Fraction(_next_down(g)) < exact


def test_nearest_sub_div_match_numpy_fp32():
    pairs = _pairs(20000, 14)
    a = np.array([p[0] for p in pairs], np.float32)
    b = np.array([p[1] for p in pairs], np.float32)
    b = np.where(b == 0, np.float32(5.0), b)
    np.testing.assert_array_equal(oracle.fp_op(a, b, "sub", up=False).view(np.uint32),
                                  (a - b).view(np.uint32))
    np.testing.assert_array_equal(oracle.fp_op(a, b, "div", up=False).view(np.uint32),
                                  (a / b).view(np.uint32))
