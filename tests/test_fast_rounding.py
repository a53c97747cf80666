"""The quantize kernel's divide-free code path, restated on the host with exact rational
arithmetic and checked against the oracle's IEEE-divide-then-rint codes (CPU only).

For a group with stored scale s and zero z the kernel takes rcp = 1/s correctly rounded
to float32, and r_lo / r_hi = the float32 values 8 units in the last place below / above
it.  For an element x it forms d = fl(x - z) and the two fused multiply-adds
fma(d, r_lo, 1.5 * 2^23) and fma(d, r_hi, 1.5 * 2^23), whose low bits are d * r_lo and
d * r_hi rounded to the nearest integer (ties to even).  Equal results are taken as the
code; otherwise the element is redone with the IEEE divide.  The claim behind it: the
exact products bracket fl(d / s), and rounding is monotone.  Here float32 rounding and
the fused operations are evaluated exactly (fractions), so a bracket that is too narrow,
a wrong magic constant, or a code above qmax shows up as a mismatch.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from bit_mixed_precision_channel_b200 import synthetic as syn

F16, BF16 = oracle.F16, oracle.BF16
MAGIC = Fraction(12582912)  # 1.5 * 2^23
LO_OK, HI_OK = Fraction(2) ** -100, Fraction(2) ** 100


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


def _rint(v: Fraction) -> int:
    r = v.numerator // v.denominator
    fr = v - r
    if fr > Fraction(1, 2) or (fr == Fraction(1, 2) and r % 2 == 1):
        r += 1
    return r


def _ulps(v: Fraction, n: int) -> Fraction:
    """The float32 n units in the last place away from the positive float32 v."""
    b = np.array([float(v)], dtype=np.float32).view(np.uint32)[0]
    return Fraction(float(np.array([b + np.uint32(n) if n >= 0 else b - np.uint32(-n)],
                                   dtype=np.uint32).view(np.float32)[0]))


def _brackets(scale: Fraction):
    """(r_lo, r_hi) as the kernel sets them, or None when it sends the group to the divide."""
    if scale == 0:
        return Fraction(0), Fraction(0)
    if not (LO_OK <= scale <= HI_OK):
        return None
    rcp = _round_f32(1 / scale)
    return _ulps(rcp, -8), _ulps(rcp, 8)


def _exact_code(x, zero, scale, qmax):
    if scale == 0:
        return 0
    q = _round_f32(_round_f32(x - zero) / scale)  # the IEEE divide, then rint, clamp
    return min(max(_rint(q), 0), qmax)


def _kernel_code(x: Fraction, zero: Fraction, scale: Fraction, qmax: int):
    """(code, took_fast_path)."""
    br = _brackets(scale)
    if br is None:
        return _exact_code(x, zero, scale, qmax), False
    r_lo, r_hi = br
    d = _round_f32(x - zero)
    lo = _round_f32(d * r_lo + MAGIC) - MAGIC  # one rounding: fma
    hi = _round_f32(d * r_hi + MAGIC) - MAGIC
    if lo == hi:
        assert 0 <= lo <= qmax, "the fast path produced a code outside [0, qmax]"
        return int(lo), True
    return _exact_code(x, zero, scale, qmax), False


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
    checked = fast = 0
    for g in _groups(rng, 40, 32, dtype):
        codes, sb, zb = oracle.quant_group(g, bits, dtype)
        scale = Fraction(oracle.value(sb, dtype))
        zero = Fraction(oracle.value(zb, dtype))
        xs = [Fraction(float(v)) for v in oracle.values(g, dtype)]
        for x, want in zip(xs, codes):
            got, took = _kernel_code(x, zero, scale, qmax)
            assert got == int(want), (bits, float(scale), float(x))
            fast += took
            checked += 1
    assert checked > 1000 and fast > 0.95 * checked


@pytest.mark.parametrize("seed", range(4))
def test_brackets_hold_the_rounded_quotient(seed):
    """d * r_lo <= fl(d / s) <= d * r_hi for scales across the fast range, including scales
    whose reciprocal sits next to a power of two (the ulp changes there)."""
    rng = np.random.default_rng(seed)
    scales = [Fraction(float(np.float32(v))) for v in 10.0 ** rng.uniform(-25, 25, 200)]
    scales += [Fraction(2) ** e * (1 + Fraction(k, 2 ** 23)) for e in (-60, -3, 0, 7, 60) for k in (-1, 0, 1, 2)]
    for s in scales:
        r_lo, r_hi = _brackets(s)
        for d in (Fraction(float(np.float32(v))) for v in rng.uniform(0, 15, 8) * float(s)):
            q = _round_f32(d / s)
            assert d * r_lo <= q <= d * r_hi


def test_exact_ties_take_the_divide():
    """x - zero = (k + 1/2) * scale exactly: the fast path must not decide, and the
    divide rounds the tie to even."""
    for scale in (Fraction(1), Fraction(3, 8), Fraction(5, 1024)):
        for k in range(15):
            x = Fraction(2 * k + 1, 2) * scale
            got, took = _kernel_code(x, Fraction(0), scale, 15)
            assert not took
            assert got == (k if k % 2 == 0 else k + 1)


def test_zero_and_out_of_range_scales():
    assert _brackets(Fraction(0)) == (0, 0)
    assert _kernel_code(Fraction(0), Fraction(0), Fraction(0), 3) == (0, True)
    assert _brackets(Fraction(2) ** -101) is None and _brackets(Fraction(2) ** 101) is None
