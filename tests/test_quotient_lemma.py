"""The one-step e4m3 quotient of bf16 values (CPU).

The epilogue divides bf16 inputs by the e4m3 scale with one corrected
Markstein step: q0 = RN(x y), r = x - q0 s, q1 = RN(q0 + r y), y = RN(1/s).
q1 can differ from the IEEE quotient RN(x / s) in its last bit; the claim is
that its e4m3 byte never does when x has at most 8 significant bits.  The
argument reduces that to an integer statement:

    for every 24-bit significand S and every point m next to an e4m3
    rounding midpoint (m = Im * 2^e with Im odd), S * Im is at least 4 away
    from every integer with at most 8 significant bits,

with one exception (S = 2^24 - 1 next to the midpoint 2^-10), which is
checked by exact evaluation of the two steps.  This file checks both parts
by brute force; the GPU suite compares the device arithmetic itself with
IEEE division for every bf16 value over whole binades of scales.
"""
from fractions import Fraction as F

import numpy as np
import pytest


def _e4m3_values():
    """Positive finite e4m3 (OCP E4M3FN) values: 7 subnormals k 2^-9, then
    significands 8..15 / 8 for exponents -6..8, 448 the largest."""
    vals = [F(k, 512) for k in range(1, 8)]
    for e in range(-6, 9):
        for m in range(8, 16):
            v = F(m, 8) * F(2) ** e
            if v <= 448:
                vals.append(v)
    return vals


def _binade(v: F) -> int:
    e = v.numerator.bit_length() - v.denominator.bit_length()
    while F(2) ** e > v:
        e -= 1
    while F(2) ** (e + 1) <= v:
        e += 1
    return e


def _fp32_ulp_above(v: F) -> F:
    return F(2) ** (_binade(v) - 23)


def _fp32_ulp_below(v: F) -> F:
    e = _binade(v)
    return F(2) ** (e - 24) if v == F(2) ** e else F(2) ** (e - 23)


def _odd_significand(v: F) -> int:
    """Im odd with v = Im * 2^k."""
    n, d = v.numerator, v.denominator
    assert d & (d - 1) == 0
    while n % 2 == 0:
        n //= 2
    return n


def _neighbour_points():
    """Odd integer significands of m = M +- half the fp32 spacing at M, for
    every e4m3 rounding midpoint M (including the one between 0 and the
    smallest subnormal)."""
    vals = [F(0)] + _e4m3_values()
    mids = [(a + b) / 2 for a, b in zip(vals, vals[1:])]
    pts = {}
    for M in mids:
        for sign, half in ((+1, _fp32_ulp_above(M) / 2), (-1, _fp32_ulp_below(M) / 2)):
            pts[(M, sign)] = _odd_significand(M + sign * half)
    return pts


def test_midpoints_have_at_most_five_bits_and_the_neighbours_the_stated_form():
    pts = _neighbour_points()
    for (M, sign), im in pts.items():
        mp = _odd_significand(M)
        assert mp.bit_length() <= 5
        k = (im - sign) // mp
        assert im == mp * k + sign and k & (k - 1) == 0
        assert 20 <= k.bit_length() - 1 <= 25


def _distance_to_8_bit_integers(p: np.ndarray, out: np.ndarray) -> np.ndarray:
    """Distance from each positive integer p (< 2^53) to the nearest integer
    with at most 8 significant bits, written into `out`."""
    _, ex = np.frexp(p.astype(np.float64))  # p in [2^(ex-1), 2^ex)
    unit = np.left_shift(np.int64(1), np.maximum(ex - 8, 0).astype(np.int64))
    np.bitwise_and(p, unit - 1, out=out)
    np.minimum(out, unit - out, out=out)
    return out


def test_no_scale_significand_puts_an_8_bit_numerator_next_to_an_e4m3_midpoint():
    S = np.arange(1 << 23, 1 << 24, dtype=np.int64)
    p = np.empty_like(S)
    d = np.empty_like(S)
    exception = _neighbour_points()[(F(1, 1024), +1)]
    worst = []
    for im in sorted(set(_neighbour_points().values())):  # many midpoints share one
        np.multiply(S, np.int64(im), out=p)
        _distance_to_8_bit_integers(p, d)
        found = [(int(S[i]), int(d[i])) for i in np.nonzero(d < 4)[0]]
        if im == exception:
            assert found == [((1 << 24) - 1, 1)], found
            d[-1] = 1 << 40
        else:
            assert found == [], (im, found[:4])
        worst.append(int(d.min()))
    # the margin is wide: every other case stays more than 2^15 units away
    assert min(worst) > 1 << 15, min(worst)


def _rn32(v: F) -> F:
    """Round to the nearest fp32, ties to even (normal range)."""
    if v == 0:
        return F(0)
    a = abs(v)
    u = F(2) ** (_binade(a) - 23)
    q = a / u
    n = q.numerator // q.denominator
    rem = q - n
    if rem > F(1, 2) or (rem == F(1, 2) and n % 2 == 1):
        n += 1
    return (1 if v > 0 else -1) * n * u


def _e4m3_round(v: F) -> F:
    a = abs(v)
    u = F(1, 512) if a < F(1, 64) else F(2) ** (_binade(a) - 3)
    q = a / u
    n = q.numerator // q.denominator
    rem = q - n
    if rem > F(1, 2) or (rem == F(1, 2) and n % 2 == 1):
        n += 1
    return (1 if v >= 0 else -1) * min(n * u, F(448))


def _one_step(x: F, s: F) -> F:
    y = _rn32(1 / s)
    q0 = _rn32(x * y)
    r = x - q0 * s  # exact in one fused multiply-add
    return _rn32(q0 + r * y)


@pytest.mark.parametrize("e", [-64, -30, -5, 0, 7, 20, 63])
def test_the_exceptional_scale_rounds_like_ieee(e):
    """s = 2^e (1 - 2^-24), x = +-2^(e-10): x / s sits just above the fp32
    midpoint next to 2^-10; the one-step quotient still rounds the same way."""
    s = F(2) ** e * (1 - F(1, 1 << 24))
    for x in (F(2) ** (e - 10), -(F(2) ** (e - 10))):
        z = x / s
        q1, ref = _one_step(x, s), _rn32(z)
        assert q1 == ref
        assert _e4m3_round(q1) == _e4m3_round(ref) != 0


def _near_midpoint_cases(n: int, seed: int):
    """(x, s) with x a bf16 value and s an fp32 scale within 3 ulp of x / M
    for an e4m3 midpoint M: x / s then lies within a few fp32 ulp of M."""
    rng = np.random.default_rng(seed)
    mids = sorted({M for (M, _) in _neighbour_points()})
    for _ in range(n):
        x = F(int(rng.integers(128, 256)), 128) * F(2) ** int(rng.integers(-20, 21))
        M = mids[int(rng.integers(len(mids)))]
        s0 = _rn32(x / M)
        for k in range(-3, 4):
            yield x, s0 + k * F(2) ** (_binade(s0) - 23)


def test_one_step_matches_ieee_bytes_next_to_midpoints():
    """Exact evaluation where it matters: x / s within a few fp32 ulp of an
    e4m3 midpoint.  The uncorrected q0 gets some of these wrong; one
    corrected step gets none wrong."""
    wrong0 = 0
    for x, s in _near_midpoint_cases(200, 7):
        ref = _e4m3_round(_rn32(x / s))
        assert _e4m3_round(_one_step(x, s)) == ref, (x, s)
        wrong0 += _e4m3_round(_rn32(x * _rn32(1 / s))) != ref
    assert wrong0 > 0
