"""Pins of the oracle's 4-bit codec against facts that do not come from it.

* An exact-arithmetic restatement: every fp32/fp16 rounding is redone on
  Python Fractions with a hand-written round-to-nearest-even, so the numpy
  quantizer is checked bit for bit by arithmetic it does not share.
* The closed-form special cases of an asymmetric min/scale code (constant
  group, exactly affine group, two-valued group, -0).
* The error bound of round-to-nearest on a 15-step grid: |x - x_hat| <= scale/2
  plus the rounding of the stored scale and of the fp16 result.
* Pack/unpack identity on every byte value.

Format: "FlexGen研究学术报告", section 三(C) (groups of 64 contiguous elements,
asymmetric, 4 bits, fp16 before compute).
"""
from fractions import Fraction

import numpy as np
import pytest

from oracle import q64

F32 = (24, -126)   # significand bits incl. the hidden one, minimum normal exponent
F16 = (11, -14)


def round_rne(x: Fraction, fmt) -> Fraction:
    """Round an exact rational to the nearest value of a binary format
    (subnormals included, no overflow handling), ties to even."""
    if x == 0:
        return Fraction(0)
    p, emin = fmt
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, emin)
    quantum = Fraction(2) ** (e - (p - 1))
    t = a / quantum
    n = t.numerator // t.denominator
    rem = t - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return sign * n * quantum


def exact_quantize_group(xs):
    """The quantizer restated with exact rationals; returns (codes, m16, s16)
    as Python values."""
    vals = [Fraction(float(v)) for v in xs]
    mn, mx = min(vals), max(vals)
    s16 = round_rne(round_rne(round_rne(mx - mn, F32) / 15, F32), F16)
    m16 = mn  # fp16 input, exact
    codes = []
    for v in vals:
        if s16 == 0:
            codes.append(0)
            continue
        r = round_rne(round_rne(v - m16, F32) / s16, F32)
        n = r.numerator // r.denominator
        rem = r - n
        if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
            n += 1
        codes.append(min(max(n, 0), 15))
    return codes, m16, s16


def exact_dequant(code, m16, s16):
    return round_rne(round_rne(round_rne(code * s16, F32) + m16, F32), F16)


def _groups(rng, count):
    """Random fp16 groups over many magnitudes, plus awkward ones."""
    out = []
    for i in range(count):
        scale = 10.0 ** rng.uniform(-7, 4)
        g = (rng.standard_normal(64) * scale + rng.standard_normal() * scale).astype(np.float16)
        out.append(g)
    out.append(np.full(64, 0.5, np.float16))
    out.append(np.array([-0.0] * 32 + [0.0] * 32, np.float16))
    sub = (np.arange(64) * 2.0 ** -24).astype(np.float16)  # subnormal ramp
    out.append(sub)
    out.append(np.linspace(-32768, 32768, 64).astype(np.float16))  # the documented input range
    return out


def test_quantizer_matches_exact_rational_restatement(rng):
    for g in _groups(rng, 60):
        codes, m16, s16 = q64.quantize(g)
        q = q64.unpack(codes)
        ec, em, es = exact_quantize_group(g)
        assert Fraction(float(m16[0])) == em
        assert Fraction(float(s16[0])) == es
        assert list(q) == ec
        deq = q64.dequantize(codes, m16, s16)
        for qi, di in zip(ec, deq):
            assert Fraction(float(di)) == exact_dequant(qi, em, es)


def test_error_bound_half_scale(rng):
    """|x - x_hat| <= s/2 + 15|s_exact - s16| + half an fp16 ulp of x_hat."""
    for g in _groups(rng, 200):
        c, m, s = q64.quantize(g)
        xh = q64.dequantize(c, m, s).astype(np.float64)
        x = g.astype(np.float64)
        s16 = float(s[0])
        s_exact = (x.max() - x.min()) / 15.0
        ulp16 = np.spacing(np.abs(xh).astype(np.float16)).astype(np.float64)
        bound = s16 / 2 + 15 * abs(s_exact - s16) + ulp16 / 2 + 1e-30
        bound = bound + 4 * np.spacing(np.float32(np.abs(x).max())).astype(np.float64)
        assert np.all(np.abs(x - xh) <= bound)


def test_constant_group_scale_zero():
    g = np.full(64, -3.25, np.float16)
    c, m, s = q64.quantize(g)
    assert s[0] == 0 and np.all(c == 0) and m[0] == np.float16(-3.25)
    assert np.array_equal(q64.dequantize(c, m, s), g)


def test_affine_group_recovers_codes(rng):
    """x = m + k s with s a power of two: the codes are exactly k."""
    k = rng.integers(0, 16, 64)
    k[0], k[1] = 0, 15
    g = (np.float32(-1.0) + k.astype(np.float32) * np.float32(0.125)).astype(np.float16)
    c, m, s = q64.quantize(g)
    assert float(s[0]) == 0.125 and float(m[0]) == -1.0
    assert np.array_equal(q64.unpack(c), k.astype(np.uint8))
    assert np.array_equal(q64.dequantize(c, m, s), g)


def test_two_valued_group():
    g = np.array([0.3, -1.7] * 32, np.float16)
    q = q64.unpack(q64.quantize(g)[0])
    assert set(q.tolist()) == {0, 15}
    assert np.array_equal(q[0::2], np.full(32, 15)) and np.array_equal(q[1::2], np.zeros(32))


def test_negative_zero_min_is_canonical():
    g = np.array([-0.0] + [1.0] * 63, np.float16)
    _, m, _ = q64.quantize(g)
    assert m.view(np.uint16)[0] == 0


def test_min_reconstructs_exactly(rng):
    for g in _groups(rng, 50):
        c, m, s = q64.quantize(g)
        xh = q64.dequantize(c, m, s)
        i = int(np.argmin(g.astype(np.float32)))
        assert float(xh[i]) == float(g[i]) or (float(xh[i]) == 0 and float(g[i]) == 0)


def test_pack_unpack_identity():
    allb = np.arange(256, dtype=np.uint8)
    assert np.array_equal(q64.pack(q64.unpack(allb)), allb)
    q = q64.unpack(allb)
    assert np.array_equal(q[0::2], allb & 15) and np.array_equal(q[1::2], allb >> 4)


def test_groups_follow_memory_order(rng):
    """Each run of 64 contiguous elements is its own group."""
    x = rng.standard_normal(256).astype(np.float16)
    x[64:128] *= 100
    c, m, s = q64.quantize(x)
    for gi in range(4):
        c1, m1, s1 = q64.quantize(x[64 * gi:64 * gi + 64])
        assert np.array_equal(c[32 * gi:32 * gi + 32], c1)
        assert m[gi] == m1[0] and s[gi] == s1[0]


def test_input_range_limit():
    """The format's input domain is |x| <= 2^15: a group spanning the whole
    fp16 range rounds its scale up far enough that 15*scale + min overflows
    fp16, so such inputs are outside the documented range."""
    g = np.linspace(-65504, 65504, 64).astype(np.float16)
    xh = q64.roundtrip(g)
    assert np.isinf(xh[-1])
    g = np.linspace(-32768, 32768, 64).astype(np.float16)
    assert np.all(np.isfinite(q64.roundtrip(g)))


def test_rejects_ragged_length():
    with pytest.raises(ValueError):
        q64.quantize(np.zeros(65, np.float16))
