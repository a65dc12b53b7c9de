"""Oracle pins for the 8-bit and 4-bit block quantisers.

Independent checks: exact rational rounding (fractions.Fraction) for every
fp16 scale input, the per-element error bound, exact round trips of scaled
integers, zero blocks, and hand-worked ties, sign and packing cases.
"""
from fractions import Fraction

import numpy as np
import pytest

from oracle import (q8_scale, q4_scale, quantize_q8, quantize_q4, dequantize_q8, dequantize_q4,
                    unpack_q4, quantize_kv, dequantize_kv, round_half_away)


# --- exact rational rounding to an IEEE binary format (independent of numpy) --------------
def _round_to_format(x: Fraction, p: int, emin: int) -> Fraction:
    """Round-to-nearest-even of a rational to precision p (incl. the hidden bit)
    with minimum normal exponent emin (gradual underflow).  No overflow handling
    is needed for the values used here."""
    if x == 0:
        return Fraction(0)
    s = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = Fraction(2) ** (max(e, emin) - (p - 1))
    n = a / ulp
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return s * fl * ulp


def _fp32(x):
    return _round_to_format(x, 24, -126)


def _fp16(x):
    return _round_to_format(x, 11, -14)


def _all_positive_finite_fp16():
    bits = np.arange(0x0001, 0x7C00, dtype=np.uint16)
    return bits.view(np.float16)


def test_q8_scale_exhaustive_against_exact_rationals():
    amax = _all_positive_finite_fp16()
    d = q8_scale(amax)
    for a, got in zip(amax.tolist(), d.astype(np.float64).tolist()):
        want = _fp16(_fp32(Fraction(a) / 127))
        assert Fraction(got) == want, (a, got, float(want))


def test_q4_scale_exhaustive_against_exact_rationals():
    m = _all_positive_finite_fp16()
    for sign in (1, -1):
        d = q4_scale((sign * m.astype(np.float32)).astype(np.float16))
        for a, got in zip(m.tolist(), d.astype(np.float64).tolist()):
            want = _fp16(Fraction(sign * a) / -8)
            assert Fraction(got) == want


def test_round_half_away():
    q = np.array([2.5, -2.5, 0.5, -0.5, 1.49999988079071, 2.4, -2.6, 0.0])
    assert round_half_away(q).tolist() == [3, -3, 1, -1, 1, 2, -3, 0]


def _blocks(seed, n, scale=1.0, outliers=False):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, 32)) * scale
    if outliers:
        x[:, rng.integers(0, 32, size=4)] *= 10
    return x.astype(np.float16)


@pytest.mark.parametrize("scale,outliers", [(1.0, False), (1.0, True), (1e-2, False), (300.0, True)])
def test_q8_error_bound(scale, outliers):
    x = _blocks(1, 4000, scale, outliers)
    c, d = quantize_q8(x)
    xh = dequantize_q8(c, d)
    normal = np.abs(d.astype(np.float64)) >= 2.0 ** -14
    assert normal.all()
    err = np.abs(x.astype(np.float64) - xh)
    assert (err <= np.abs(d.astype(np.float64))[:, None] / 2).all()
    assert np.abs(c.astype(int)).max() <= 127


@pytest.mark.parametrize("scale,outliers", [(1.0, False), (1.0, True), (1e-2, False), (300.0, True)])
def test_q4_error_bound(scale, outliers):
    x = _blocks(2, 4000, scale, outliers)
    p, d = quantize_q4(x)
    xh = dequantize_q4(p, d)
    assert (np.abs(d.astype(np.float64)) >= 2.0 ** -14).all()
    err = np.abs(x.astype(np.float64) - xh)
    assert (err <= np.abs(d.astype(np.float64))[:, None]).all()
    # the largest-magnitude element maps to code -8 exactly (all 16 levels used)
    u = unpack_q4(p) + 8
    idx = np.argmax(np.abs(x), axis=-1)
    assert (u[np.arange(len(x)), idx] == 0).all()


def test_q8_scaled_integer_round_trip_is_exact():
    rng = np.random.default_rng(3)
    for k in range(-6, 5):
        c = rng.integers(-127, 128, size=(50, 32))
        c[:, 0] = 127 * rng.choice([-1, 1], size=50)           # amax = 127 * 2^k
        x = (c * 2.0 ** k).astype(np.float16)
        codes, d = quantize_q8(x)
        assert (d.astype(np.float64) == 2.0 ** k).all()
        assert (codes.astype(int) == c).all()
        assert (dequantize_q8(codes, d) == x.astype(np.float64)).all()


def test_q4_scaled_integer_round_trip_is_exact():
    rng = np.random.default_rng(4)
    for k in range(-6, 5):
        c = rng.integers(-7, 8, size=(50, 32))
        c[:, 5] = -8                                             # m = -8 * 2^k -> d = 2^k
        x = (c * 2.0 ** k).astype(np.float16)
        p, d = quantize_q4(x)
        assert (d.astype(np.float64) == 2.0 ** k).all()
        assert (unpack_q4(p) == c).all()


def test_zero_block():
    x = np.zeros((3, 32), np.float16)
    c, d = quantize_q8(x)
    assert (c == 0).all() and (d == 0).all()
    p, d4 = quantize_q4(x)
    assert (d4 == 0).all() and (p == 0x88).all()               # code 0 -> nibble 8
    assert (dequantize_q4(p, d4) == 0).all()


def test_q8_hand_worked_ties():
    # amax = 127 -> d = 1 exactly; 2.5 -> 3 and -2.5 -> -3 (ties away from zero)
    x = np.zeros(32, np.float16)
    x[0], x[1], x[2], x[3], x[4] = 127, 2.5, -2.5, 0.5, -1.5
    c, d = quantize_q8(x)
    assert float(d) == 1.0
    assert c[:5].tolist() == [127, 3, -3, 1, -2]


def test_q4_hand_worked_sign_tie_break_and_packing():
    # m = -8 at index 0 -> d = -8 / -8 = +1; element values map straight to codes
    x = np.zeros(32, np.float16)
    x[0] = -8
    x[1], x[2], x[16], x[17], x[31] = 7, 2.5, -3, 1.5, 4
    p, d = quantize_q4(x)
    assert float(d) == 1.0
    u = [0] * 32
    for j, c in enumerate([-8, 7, 3, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0,
                           -3, 2, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 4]):
        u[j] = c + 8
    want = [u[i] | (u[i + 16] << 4) for i in range(16)]
    assert p.tolist() == want
    assert p.tolist()[:3] == [0x50, 0xAF, 0x8B]

    # +a and -a both of largest magnitude: the lower index wins
    y = np.zeros(32, np.float16)
    y[3], y[10] = -4, 4
    p, d = quantize_q4(y)
    assert float(d) == 0.5                                       # m = -4 -> d = 0.5
    c = unpack_q4(p)
    assert c[3] == -8 and c[10] == 7                            # +8 clamps to +7, error = |d|
    y[3], y[10] = 4, -4
    p, d = quantize_q4(y)
    assert float(d) == -0.5
    c = unpack_q4(p)
    assert c[3] == -8 and c[10] == 7


def test_subnormal_scales_are_deterministic():
    # tiny blocks: scales fall in the fp16 subnormal range; codes stay in range
    x = (_blocks(5, 500).astype(np.float64) * 1e-6).astype(np.float16)
    c, d = quantize_q8(x)
    assert np.abs(c.astype(int)).max() <= 127
    p, d4 = quantize_q4(x)
    assert unpack_q4(p).min() >= -8 and unpack_q4(p).max() <= 7


@pytest.mark.parametrize("bits", [16, 8, 4])
def test_kv_layout_round_trip(bits):
    rng = np.random.default_rng(6)
    x = rng.standard_normal((5, 3, 64)).astype(np.float16)
    codes, scales = quantize_kv(x, bits)
    if bits == 16:
        assert scales is None and (codes == x).all()
    else:
        assert scales.shape == (5, 3, 2)
        assert codes.shape == (5, 3, 64 if bits == 8 else 32)
        # block b of (t, h) is elements [32b, 32b + 32) of that row
        flat = x.reshape(-1, 32)
        c2, d2 = (quantize_q8 if bits == 8 else quantize_q4)(flat)
        assert (scales.reshape(-1) == d2).all()
    xh = dequantize_kv(codes, scales, bits)
    tol = {16: 0.0, 8: 0.5, 4: 1.0}[bits]
    if bits != 16:
        bound = np.repeat(np.abs(scales.astype(np.float64)), 32, axis=-1) * tol
        assert (np.abs(xh - x.astype(np.float64)) <= bound).all()
    else:
        assert (xh == x.astype(np.float64)).all()
