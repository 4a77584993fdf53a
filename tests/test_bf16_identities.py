"""The two bf16 identities the HF-mode kernels rely on when they replace
"fp32 operation, then round to bf16" by one packed bf16x2 operation
(mul.rn.bf16x2 / add.rn.bf16x2, each rounding the exact result once):

  * the product of two bf16 values is exact in fp32, so rounding the fp32
    product to bf16 is rounding the exact product once;
  * rounding an fp32 sum of two bf16 values to bf16 gives the exact sum
    rounded once to bf16 (the fp32 sum is inexact only for exponent gaps of
    16 or more, and then lies far from every bf16 rounding midpoint).

Checked here on random pairs, with exact rational arithmetic as the
reference."""
from fractions import Fraction

import numpy as np


def _bf16_bits_rne(x32):
    b = np.asarray(x32, np.float32).view(np.uint32).astype(np.uint64)
    return (((b + 0x7FFF + ((b >> 16) & 1)) >> 16) & 0xFFFF).astype(np.uint32)


def _bf16_value(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32)


def _round_exact_to_bf16(q):
    """Fraction -> bf16 bits, round to nearest even (finite, normal range)."""
    if q == 0:
        return 0
    neg = q < 0
    q = abs(q)
    e = q.numerator.bit_length() - q.denominator.bit_length()
    while Fraction(2) ** e > q:
        e -= 1
    while Fraction(2) ** (e + 1) <= q:
        e += 1
    ulp = Fraction(2) ** (e - 7)
    units = q / ulp
    n = units.numerator // units.denominator
    rem = units - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    v = float(n * ulp) * (-1.0 if neg else 1.0)
    return int(_bf16_bits_rne(np.float32(v)))


def _pairs(rng, n, max_gap):
    a = _bf16_value(rng.integers(0, 1 << 16, n))
    keep = np.isfinite(a) & (np.abs(a) > 1e-30) & (np.abs(a) < 1e30)
    a = a[keep]
    gap = rng.integers(0, max_gap + 1, a.size).astype(np.float64)
    mant = rng.integers(0x80, 0x100, a.size) / 128.0
    sign = np.where(rng.random(a.size) < 0.5, -1.0, 1.0)
    b = (sign * mant * np.abs(a.astype(np.float64)) * 2.0 ** -gap).astype(np.float32)
    return a, _bf16_value(_bf16_bits_rne(b))


def test_bf16_products_are_exact_in_fp32():
    # the kernels' products: a bf16 value times a weight or a cos / sin in [-1, 1]
    rng = np.random.default_rng(11)
    a = _bf16_value(_bf16_bits_rne(rng.standard_normal(20000) * 2.0 ** rng.integers(-40, 40, 20000)))
    b = _bf16_value(_bf16_bits_rne(rng.uniform(-1.0, 1.0, 20000)))
    exact = a.astype(np.float64) * b.astype(np.float64)
    ok = np.abs(exact) > 1e-37                # stay clear of the fp32 subnormal range
    assert ok.sum() > 19000
    assert np.array_equal(exact[ok], (a * b).astype(np.float64)[ok])


def test_fp32_sum_then_round_is_one_bf16_rounding():
    rng = np.random.default_rng(12)
    a, b = _pairs(rng, 6000, 30)
    via_fp32 = _bf16_bits_rne((a + b).astype(np.float32))
    inexact = 0
    for x, y, got in zip(a.tolist(), b.tolist(), via_fp32.tolist()):
        s = Fraction(x) + Fraction(y)
        inexact += s != Fraction(float(np.float32(x) + np.float32(y)))
        assert got == _round_exact_to_bf16(s), (x, y)
    assert inexact > 1000                  # the hard case (inexact fp32 sums) is well covered
