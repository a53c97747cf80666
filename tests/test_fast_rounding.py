"""The quantize kernel's divide-free code path, restated on the host with exact rational
arithmetic and checked against the oracle's IEEE-divide-then-rint codes (CPU only).

The kernel computes t = fma(d, rcp, 1.5 * 2^23) with d = fl(x - zero) and rcp an
approximate reciprocal of the scale (within one float32 ulp), takes the code from the low
bits of t, and hands the element to the IEEE divide when |fl(d * rcp - n)| is not below
1/2 - 2^-14.  Here fma and float32 rounding are evaluated exactly (fractions), with the
reciprocal set to its correctly rounded value and to the neighbours one ulp away, so a wrong
margin or a wrong claim that no code exceeds qmax shows up as a mismatch.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from bit_mixed_precision_channel_b200 import synthetic as syn

F16, BF16 = oracle.F16, oracle.BF16
MAGIC = Fraction(12582912)                      # 1.5 * 2^23
NEAR = Fraction(1, 2) - Fraction(1, 16384)      # 1/2 - 2^-14


def _round_f32(v: Fraction) -> Fraction:
    """v rounded to the nearest float32, ties to even (normal range only)."""
    if v == 0:
        return v
    sign = -1 if v < 0 else 1
    a = abs(v)
    e = a.numerator.bit_length() - a.denominator.bit_length()  # 2^e <= a < 2^(e+2)
    if a < Fraction(2) ** e:
        e -= 1
    elif a >= Fraction(2) ** (e + 1):
        e += 1
    m = a / (Fraction(2) ** (e - 23))                            # in [2^23, 2^24)
    n = m.numerator // m.denominator
    frac = m - n
    if frac > Fraction(1, 2) or (frac == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return sign * n * (Fraction(2) ** (e - 23))


def _kernel_code(x: Fraction, zero: Fraction, scale: Fraction, rcp: Fraction, qmax: int) -> int:
    d = _round_f32(x - zero)
    t = _round_f32(d * rcp + MAGIC)                 # one rounding: fma
    n = int(t - MAGIC)
    res = _round_f32(d * rcp - (t - MAGIC))         # fma(d, rcp, -(t - M))
    if abs(res) < NEAR:
        assert n <= qmax, "the fast path produced a code above qmax"
        return n
    q = _round_f32(d / scale)                       # the IEEE divide, then rint, clamp
    r = q.numerator // q.denominator
    fr = q - r
    if fr > Fraction(1, 2) or (fr == Fraction(1, 2) and r % 2 == 1):
        r += 1
    return min(max(r, 0), qmax)


def _groups(rng, n_groups, size, dtype):
    out = []
    for i in range(n_groups):
        scale = 10.0 ** rng.uniform(-3, 2)
        x = rng.standard_normal(size) * scale
        if i % 5 == 0:  # values on a coarse grid: many exact and near ties
            x = np.round(x / scale * 4) / 4 * scale
        out.append(syn.to_bits(x.astype(np.float32), dtype))
    return out


@pytest.mark.parametrize("dtype,bits", [(F16, 2), (F16, 4), (BF16, 2), (BF16, 4)])
def test_divide_free_codes_equal_the_oracle(dtype, bits):
    rng = np.random.default_rng(100 * dtype + bits)
    qmax = (1 << bits) - 1
    checked = 0
    for g in _groups(rng, 40, 32, dtype):
        codes, sb, zb = oracle.quant_group(g, bits, dtype)
        scale = Fraction(oracle.value(sb, dtype))
        zero = Fraction(oracle.value(zb, dtype))
        if scale == 0 or float(scale) < 1.17549435e-38:
            continue  # the kernel sends these groups to the IEEE divide outright
        exact_rcp = _round_f32(1 / scale)
        ulp = Fraction(2) ** (int(np.frexp(float(exact_rcp))[1]) - 24)
        xs = [Fraction(float(v)) for v in oracle.values(g, dtype)]
        for rcp in (exact_rcp - ulp, exact_rcp, exact_rcp + ulp):
            got = [_kernel_code(x, zero, scale, rcp, qmax) for x in xs]
            assert got == [int(c) for c in codes], (bits, float(scale), float(rcp))
            checked += len(xs)
    assert checked > 2000


def test_exact_ties_take_the_divide():
    """x - zero = (k + 1/2) * scale exactly: the fast path must not decide."""
    scale, zero = Fraction(1), Fraction(0)
    for k in range(15):
        x = Fraction(2 * k + 1, 2)
        d = _round_f32(x - zero)
        t = _round_f32(d * 1 + MAGIC)
        res = _round_f32(d - (t - MAGIC))
        assert not abs(res) < NEAR
        assert _kernel_code(x, zero, scale, Fraction(1), 15) == (k if k % 2 == 0 else k + 1)
