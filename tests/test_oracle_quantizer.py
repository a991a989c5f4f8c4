"""Pins of the oracle's group quantizer and bit packing.

The pages ("Kuantisasi KV cache mengganggu attention ...", section
"Granularitas kuantisasi menentukan nilai yang berbagi scale"; tag-index
teaser "... Biaya Rekonstruksi") fix a group-wise mapping with a scale and a
zero point; the formula is the plain min/max reading.  What pins it here,
independently of the oracle's own arithmetic:

* invariants on every element, checked in exact rational / fp64 arithmetic:
  the code grid covers the group, codes are in range, and the reconstruction
  error is at most scale/2 (plus the fp32 rounding of the two IEEE steps);
* brute force: the chosen code is the nearest grid point among all 2^b codes;
* closed forms: groups already on a representable grid round-trip exactly;
  constant groups give scale 0 and exact reconstruction;
* hand-written packing examples and pack/unpack round trips.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle


def f16val(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def _groups(seed, rows, n):
    r = np.random.default_rng(seed)
    blocks = [
        r.standard_normal((rows, n)),
        r.standard_normal((rows, n)) * 10 + 3,
        r.standard_normal((rows, n)) * 1e-3,
        r.standard_normal((rows, n)) * 1e-6,           # fp16 subnormal scales
        r.uniform(-200, -100, (rows, n)),              # all negative
        r.uniform(1000, 1000.01, (rows, n)),           # narrow range far from 0
        r.standard_t(3, (rows, n)) * 10,               # heavy tails
    ]
    x = r.standard_normal((rows, n))
    x[:, 3] *= 40                                       # one outlier channel
    blocks.append(x)
    return np.concatenate(blocks).astype(np.float32)


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
@pytest.mark.parametrize("group", [32, 64, 128])
def test_invariants(bits, group):
    x = _groups(100 + bits * 7 + group, 200, group)
    s, z, c = oracle.quantize_rows(x, group, bits)
    sf, zf = f16val(s)[:, 0], f16val(z)[:, 0]
    x64 = x.astype(np.float64)
    qmax = 2 ** bits - 1
    mn, mx = x64.min(1), x64.max(1)
    assert np.all(c <= qmax)
    assert np.all(zf <= mn)                                  # zero rounded down
    assert np.all(zf + qmax * sf >= mx)                      # grid covers the group
    # zero is the largest fp16 not above the minimum
    up = np.nextafter(z[:, 0].view(np.float16), np.float16(np.inf)).astype(np.float64)
    assert np.all((up > mn) | (z[:, 0] == 0x7BFF))
    xhat = oracle.dequantize_rows(c, s, z, group).astype(np.float64)
    err = np.abs(x64 - xhat)
    ulp = np.spacing(np.abs(xhat).astype(np.float32)).astype(np.float64)
    bound = sf[:, None] * (0.5 + 2.0 ** (bits - 23)) + 0.5 * ulp
    assert np.all(err <= bound)


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
def test_nearest_code_brute_force(bits):
    group = 32
    x = _groups(300 + bits, 60, group)
    s, z, c = oracle.quantize_rows(x, group, bits)
    sf, zf = f16val(s)[:, 0], f16val(z)[:, 0]
    grid = np.arange(2 ** bits, dtype=np.float64)
    for r in range(x.shape[0]):
        if sf[r] == 0:
            assert np.all(c[r] == 0)
            continue
        pts = grid * sf[r] + zf[r]                               # exact in fp64
        for j in range(group):
            d = np.abs(pts - float(x[r, j]))
            best = d.min()
            # the fp32 evaluation of (x - zero)/scale may move a near-tie by a
            # few ulps of the quotient (at most 2^(bits-23) grid steps)
            assert d[c[r, j]] <= best + sf[r] * 2.0 ** (bits - 22), (r, j)


def test_tiny_groups_enumerated():
    """Groups of up to 4 values at 1 and 2 bits: every code vector is tried;
    the oracle's vector minimises the worst element error for its metadata."""
    r = np.random.default_rng(5)
    for bits in (1, 2):
        for n in (1, 2, 3, 4):
            for _ in range(200):
                x = (r.standard_normal(n) * r.choice([0.01, 1, 100])).astype(np.float32)
                s, z, c = oracle.quantize_rows(x[None], n, bits)
                sf, zf = float(f16val(s)[0, 0]), float(f16val(z)[0, 0])
                best = None
                for idx in np.ndindex(*([2 ** bits] * n)):
                    e = max(abs(float(x[i]) - (idx[i] * sf + zf)) for i in range(n))
                    best = e if best is None else min(best, e)
                got = max(abs(float(x[i]) - (int(c[0, i]) * sf + zf)) for i in range(n))
                assert got <= best + sf * 2.0 ** (bits - 22) + 1e-30


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
def test_grid_groups_round_trip_exactly(bits):
    r = np.random.default_rng(40 + bits)
    qmax = 2 ** bits - 1
    for _ in range(200):
        zero = np.float16(r.integers(-64, 64) / 4.0)
        scale = np.float16(2.0 ** int(r.integers(-6, 3)))
        k = r.integers(0, qmax + 1, 32)
        k[0], k[1] = 0, qmax
        x = (float(zero) + k * float(scale)).astype(np.float32)
        assert np.all(x.astype(np.float64) == float(zero) + k * float(scale))
        s, z, c = oracle.quantize_rows(x[None], 32, bits)
        assert s[0, 0] == scale.view(np.uint16) and z[0, 0] == zero.view(np.uint16)
        np.testing.assert_array_equal(c[0], k)
        xhat = oracle.dequantize_rows(c, s, z, 32)
        np.testing.assert_array_equal(xhat[0], x)


def test_constant_groups():
    for v in (0.0, 1.5, -3.25, 1000.0):
        x = np.full((1, 32), v, np.float32)
        s, z, c = oracle.quantize_rows(x, 32, 4)
        assert s[0, 0] == 0 and np.all(c == 0)
        np.testing.assert_array_equal(oracle.dequantize_rows(c, s, z, 32), x)
    # negative zeros are stored as +0
    x = np.full((1, 32), -0.0, np.float32)
    s, z, c = oracle.quantize_rows(x, 32, 2)
    assert s[0, 0] == 0 and z[0, 0] == 0
    # a constant that fp16 cannot hold still gets a positive scale
    x = np.full((1, 32), 0.1, np.float32)
    s, z, c = oracle.quantize_rows(x, 32, 4)
    assert s[0, 0] != 0
    xhat = oracle.dequantize_rows(c, s, z, 32)
    assert np.all(np.abs(xhat - x) <= f16val(s)[0, 0] / 2 + 1e-8)


def test_pack_hand_examples():
    # nibbles 0..15: little-endian words 0x76543210, 0xFEDCBA98
    got = oracle.pack(np.arange(16), 4)
    assert got.tobytes() == bytes([0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE])
    # crumbs 0,1,2,3 repeated: every byte 0b11100100
    assert oracle.pack(np.tile(np.arange(4), 4), 2).tobytes() == bytes([0xE4] * 4)
    # alternating bits 1,0: 0x55 bytes
    assert oracle.pack(np.tile([1, 0], 16), 1).tobytes() == bytes([0x55] * 4)
    # bytes are stored as-is
    assert oracle.pack(np.array([1, 2, 3, 250]), 8).tobytes() == bytes([1, 2, 3, 250])


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
def test_pack_round_trip(bits):
    r = np.random.default_rng(bits)
    codes = r.integers(0, 2 ** bits, 128).astype(np.uint8)
    packed = oracle.pack(codes, bits)
    assert packed.size == 128 * bits // 8
    np.testing.assert_array_equal(oracle.unpack(packed, 128, bits), codes)


def test_scale_rounding_is_directed_not_nearest():
    """A group whose exact (max-min)/(2^b-1) lies just above an fp16 value:
    round-to-nearest would shrink the grid below the maximum; the oracle's
    upward rounding keeps it covered."""
    bits = 4
    sc = np.float16(0.5)
    mx = np.float32(float(sc) * 15 + 2.0 ** -13)      # 7.5 + tiny
    x = np.zeros(32, np.float32)
    x[0] = 0.0
    x[1] = mx
    s, z, c = oracle.quantize_rows(x[None], 32, bits)
    assert float(f16val(s)[0, 0]) * 15 >= float(mx)
    assert float(f16val(s)[0, 0]) > 0.5
    assert Fraction(float(mx)) <= Fraction(float(f16val(s)[0, 0])) * 15
