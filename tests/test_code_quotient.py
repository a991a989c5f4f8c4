"""The per-channel append forms a code as rint((x - zero) * (1 / scale)) with
both operations correctly rounded in fp32, and divides instead when a
half-integer lies within 2^-20 |q| of the product (the product is within
about 2^-22 |q| of the exact quotient, the correctly rounded quotient within
2^-24 |q|).  This checks, in IEEE fp32 on the host, that the codes equal
those of one correctly rounded division per value, on random values and on
values placed a few ulps from the rounding boundaries of every code, for
every bit width.  The kernel body itself is compared with the oracle byte
for byte by tests/test_channel_emulated.py and on the GPU."""
import numpy as np
import pytest

F = np.float32


def codes_by_reciprocal(x, zf, sf, qmax):
    a = (x - zf).astype(F)
    q = (a * (F(1.0) / sf).astype(F)).astype(F)
    fq = np.floor(q).astype(F)
    near = np.abs((q - fq).astype(F) - F(0.5)) <= (np.abs(q) * F(2.0 ** -20)).astype(F)
    q = np.where(near, (a / sf).astype(F), q)
    return np.clip(np.rint(q), 0, qmax), near


def codes_by_division(x, zf, sf, qmax):
    return np.clip(np.rint(((x - zf).astype(F) / sf).astype(F)), 0, qmax)


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
def test_reciprocal_codes_equal_division_codes(bits):
    rng = np.random.default_rng(100 + bits)
    qmax = 2 ** bits - 1
    fallbacks = 0
    for trial in range(6):
        n = 40000
        sf = F(np.float16(rng.uniform(1e-4, 4.0)))
        zf = F(np.float16(rng.normal(0.0, 2.0)))
        x_rand = (zf + rng.uniform(0, qmax + 1, n).astype(F) * sf).astype(F)
        k = rng.integers(0, qmax + 1, n).astype(F)
        x_edge = (zf + (k + F(0.5)) * sf).astype(F)
        steps = rng.integers(-3, 4, n)
        for s in range(3):                      # up to three ulps either side of the boundary
            move = np.abs(steps) > s
            x_edge = np.where(move, np.nextafter(x_edge, np.where(steps > 0, np.inf, -np.inf).astype(F)),
                              x_edge).astype(F)
        for x in (x_rand, x_edge):
            got, near = codes_by_reciprocal(x, zf, sf, qmax)
            np.testing.assert_array_equal(got, codes_by_division(x, zf, sf, qmax))
            fallbacks += int(near.sum())
    assert fallbacks > 0                        # the boundary cases do reach the division
