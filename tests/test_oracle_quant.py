"""Pins of the oracle's quantizer and 16-bit conversions (CPU only).

Each test checks the oracle against something other than itself: hand-worked
examples (tests/golden), numpy / torch conversions, brute force over all codes,
the error bound of round-to-nearest, exact recovery of on-grid inputs.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from bit_mixed_precision_channel_b200 import synthetic as syn

F16, BF16 = oracle.F16, oracle.BF16


def _bits(x, dtype):
    return syn.to_bits(np.asarray(x, np.float32), dtype)


# ----------------------------------------------------------------- 16-bit conversions

def _f16_up_numpy(x: float) -> int:
    h = np.float16(x)
    if float(h) < x:
        h = np.nextafter(h, np.float16(np.inf))
    return int(np.array(h).view(np.uint16))


def _bf16_up_torch(x: float) -> int:
    t = torch.tensor([x], dtype=torch.float64).to(torch.bfloat16)
    if float(t) < x:
        b = int(t.view(torch.int16).item()) & 0xFFFF
        b = b + 1 if b < 0x8000 else b - 1  # next bf16 toward +inf
        return b
    return int(t.view(torch.int16).item()) & 0xFFFF


def test_f16_round_up_and_nearest_match_numpy():
    rng = np.random.default_rng(1)
    xs = np.concatenate([
        rng.standard_normal(3000) * 10.0 ** rng.integers(-9, 5, 3000),
        rng.uniform(0, 1e-7, 200),            # subnormal range of fp16
        [1 / 3, 2 / 3, 0.1, 65504.0, 65000.5, 6.1e-5, -6.1e-5, 0.0]])
    for x in xs.astype(np.float32).astype(np.float64):
        assert oracle.round_up(x, F16) == _f16_up_numpy(float(x)), x
        assert oracle.round_nearest(x, F16) == int(np.array(np.float16(x)).view(np.uint16)), x


def test_bf16_round_up_and_nearest_match_torch():
    rng = np.random.default_rng(2)
    xs = rng.standard_normal(3000) * 10.0 ** rng.integers(-30, 30, 3000)
    for x in np.concatenate([xs, [1 / 3, 0.0, 1e-39]]).astype(np.float32).astype(np.float64):
        near = int(torch.tensor([float(x)], dtype=torch.float64).to(torch.bfloat16)
                   .view(torch.int16).item()) & 0xFFFF
        assert oracle.round_nearest(x, BF16) == near, x
        assert oracle.round_up(x, BF16) == _bf16_up_torch(float(x)), x


def test_values_decode_exactly():
    allbits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    f = allbits.view(np.float16).astype(np.float64)
    finite = np.isfinite(f)
    sample = np.nonzero(finite)[0][::97]
    for i in sample:
        assert oracle.value(int(allbits[i]), F16) == f[i]
    bf = torch.from_numpy(allbits.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    for i in np.nonzero(np.isfinite(bf))[0][::89]:
        assert oracle.value(int(allbits[i]), BF16) == bf[i]


# ----------------------------------------------------------------------- quantizer

def _golden():
    here = os.path.dirname(os.path.abspath(__file__))
    with open(os.path.join(here, "golden", "quant_group_examples.json")) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden(), ids=lambda c: c["name"])
def test_quant_group_hand_worked_examples(case):
    dtype = F16 if case["dtype"] == "f16" else BF16
    codes, sb, zb = oracle.quant_group(_bits(case["x"], dtype), case["bits"], dtype)
    assert codes.tolist() == case["codes"]
    assert sb == int(case["scale_bits"], 16)
    assert zb == int(case["zero_bits"], 16)
    assert oracle.value(sb, dtype) == case["scale"]
    assert oracle.value(zb, dtype) == case["zero"]


def _random_group(rng, n, dtype):
    x = rng.standard_normal(n) * rng.choice([0.01, 1.0, 30.0]) + rng.normal() * 3
    return _bits(x, dtype)


@pytest.mark.parametrize("dtype", [F16, BF16])
@pytest.mark.parametrize("bits", [2, 4])
def test_quant_group_brute_force(dtype, bits):
    """Every code is the nearest grid point (ties to even) among all 2^b codes, and the
    scale is the smallest storage value >= the fp32 quotient (mx - mn)/(2^b - 1)."""
    rng = np.random.default_rng(10 + bits + 7 * dtype)
    qmax = (1 << bits) - 1
    checked = total = 0
    for trial in range(400):
        n = int(rng.choice([2, 3, 5, 8, 32, 128]))
        xb = _random_group(rng, n, dtype)
        codes, sb, zb = oracle.quant_group(xb, bits, dtype)
        xv = oracle.values(xb, dtype)
        scale, zero = oracle.value(sb, dtype), oracle.value(zb, dtype)
        # scale: smallest 16-bit value >= fp32 quotient, computed here with numpy float32
        q32 = float(np.float32(np.float32(xv.max()) - np.float32(xv.min())) / np.float32(qmax))
        assert scale >= q32
        below = float(syn.from_bits(np.array([sb - 1], np.uint16), dtype)[0]) if sb > 0 else -1
        assert below < q32
        assert zero == xv.min()
        if scale == 0:
            assert (codes == 0).all()
            continue
        for x, c in zip(xv, codes):
            total += 1
            t = (Fraction(x) - Fraction(zero)) / Fraction(scale)
            # skip the rare elements within 1e-5 of (but not exactly on) a rounding
            # boundary, where the fp32 quotient of the definition decides; exact ties
            # are checked (they must go to the even code)
            half = int(t) + Fraction(1, 2)
            if t != half and abs(t - half) < Fraction(1, 100000):
                continue
            checked += 1
            dist = [abs(Fraction(x) - (k * Fraction(scale) + Fraction(zero))) for k in range(qmax + 1)]
            best = min(dist)
            cands = [k for k in range(qmax + 1) if dist[k] == best]
            want = cands[0] if len(cands) == 1 else [k for k in cands if k % 2 == 0][0]
            assert c == want, (x, zero, scale, c, want)
    assert checked > 0.99 * total


def test_quant_group_exact_ties_go_to_even():
    x = _bits([0.0, 0.5, 1.5, 2.5, 3.0], F16)
    codes, sb, zb = oracle.quant_group(x, 2, F16)
    assert codes.tolist() == [0, 0, 2, 2, 3]
    x4 = _bits([0.0, 0.5, 1.5, 2.5, 3.5, 4.5, 15.0], F16)
    codes4, _, _ = oracle.quant_group(x4, 4, F16)
    assert codes4.tolist() == [0, 0, 2, 2, 4, 4, 15]


@pytest.mark.parametrize("dtype", [F16, BF16])
@pytest.mark.parametrize("bits", [2, 4])
def test_quant_group_error_bound(dtype, bits):
    """|x - (code*scale + zero)| <= scale/2 + a few fp32 ulps, and the bound is nearly met."""
    rng = np.random.default_rng(20 + bits + dtype)
    worst = 0.0
    for _ in range(300):
        n = int(rng.choice([32, 128]))
        xb = _random_group(rng, n, dtype)
        codes, sb, zb = oracle.quant_group(xb, bits, dtype)
        xv = oracle.values(xb, dtype)
        s, z = oracle.value(sb, dtype), oracle.value(zb, dtype)
        xh = codes * s + z
        slack = 4 * np.spacing(np.float32(np.abs(xv).max() + abs(z) + (2 ** bits) * s)).astype(np.float64)
        err = np.abs(xv - xh)
        assert (err <= s / 2 + slack).all()
        if s > 0:
            worst = max(worst, float((err / s).max()))
    assert worst > 0.45  # a scale that were too large would never come near s/2


@pytest.mark.parametrize("dtype", [F16, BF16])
@pytest.mark.parametrize("bits", [2, 4])
def test_quant_group_recovers_grid_inputs(dtype, bits):
    """Inputs already on a power-of-two grid come back exactly: scale, zero and codes."""
    rng = np.random.default_rng(30 + bits)
    qmax = (1 << bits) - 1
    for _ in range(100):
        s = 2.0 ** int(rng.integers(-6, 3))
        mn = s * int(rng.integers(-20, 20))
        c = rng.integers(0, qmax + 1, size=32)
        lo_i, hi_i = rng.choice(32, size=2, replace=False)
        c[lo_i], c[hi_i] = 0, qmax
        x = mn + c * s
        codes, sb, zb = oracle.quant_group(_bits(x, dtype), bits, dtype)
        assert oracle.value(sb, dtype) == s
        assert oracle.value(zb, dtype) == mn
        assert (codes == c).all()
        assert np.array_equal(codes * s + mn, x)


@pytest.mark.parametrize("bits", [2, 4])
def test_quant_group_idempotent_on_its_own_output(bits):
    """Quantizing a group's dequantized values (when they are fp16 values and hit both
    ends of the range) reproduces the scale, the zero and the codes."""
    rng = np.random.default_rng(40 + bits)
    qmax = (1 << bits) - 1
    n_checked = 0
    for _ in range(500):
        xb = _random_group(rng, 32, F16)
        codes, sb, zb = oracle.quant_group(xb, bits, F16)
        s, z = oracle.value(sb, F16), oracle.value(zb, F16)
        xh = codes * s + z
        if s == 0 or codes.min() != 0 or codes.max() != qmax:
            continue
        xh16 = xh.astype(np.float16)
        if not np.array_equal(xh16.astype(np.float64), xh):
            continue  # dequantized values not representable in fp16
        if oracle.round_up(float(np.float32(xh.max() - xh.min()) / np.float32(qmax)), F16) != sb:
            continue
        codes2, sb2, zb2 = oracle.quant_group(xh16.view(np.uint16), bits, F16)
        assert (codes2 == codes).all() and sb2 == sb and zb2 == zb
        n_checked += 1
    assert n_checked > 20


def test_quant_group_constant_and_signed_zero():
    codes, sb, zb = oracle.quant_group(_bits([-2.25] * 32, F16), 2, F16)
    assert (codes == 0).all() and sb == 0 and oracle.value(zb, F16) == -2.25
    codes, sb, zb = oracle.quant_group(np.array([0x8000, 0x3C00, 0x4000], np.uint16), 2, F16)
    assert zb == 0x0000
