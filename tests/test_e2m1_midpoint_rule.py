"""The rule by which the activation quantizers decide an E2M1 code without dividing.

An FP4 code is the E2M1 rounding of the value over its block scale, the quotient rounded once to fp32
("Under the hood", "Quantization: BF16 vs NVFP4": FP4 elements with FP8 block scales; the oracle takes the
code of fl32(v / s)).  For a scale s that is a positive E4M3 value the kernels instead compare |v| - t*s,
rounded once as an fma rounds it, against +-h*s for each E2M1 midpoint t (h: half the fp32 spacing at t
on the side that matters; "<=" at the midpoints where a value exactly on t takes the lower code, "<" where it
takes the upper one; a quotient exactly halfway between t and its fp32 neighbour rounds onto t, since every
midpoint's last mantissa bit is even).
This test checks that rule, in exact rational arithmetic, against the rounded quotient for every positive
E4M3 scale at, around and between the midpoints.  It checks the mathematics the kernels rely on; the
kernels themselves are compared bit for bit with the oracle's division in the GPU tests.
"""
from fractions import Fraction as F

import numpy as np
import pytest


def _round_f32(q: F) -> F:
    """q rounded to the nearest fp32 value, ties to even (normal and subnormal range)."""
    if q == 0:
        return F(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while a >= F(2) ** (e + 1):
        e += 1
    while a < F(2) ** e:
        e -= 1
    e = max(e, -126)
    scaled = a / F(2) ** (e - 23)
    n = scaled.numerator // scaled.denominator
    rem = scaled - n
    if rem > F(1, 2) or (rem == F(1, 2) and n % 2 == 1):
        n += 1
    return sign * F(n) * F(2) ** (e - 23)


def _code_of_quotient(v: float, s: F) -> int:
    """E2M1 code of fl32(v / s): the definition."""
    q = _round_f32(F(v) / s)
    m = abs(q)
    c = (0 if m <= F(1, 4) else 1 if m < F(3, 4) else 2 if m <= F(5, 4) else 3 if m < F(7, 4)
         else 4 if m <= F(5, 2) else 5 if m < F(7, 2) else 6 if m <= 5 else 7)
    return c | 8 if c and q < 0 else c


# (midpoint t, half the fp32 spacing at t, tie rounds down onto t)
_MIDPOINTS = [(F(1, 4), F(1, 2 ** 26), True), (F(3, 4), F(1, 2 ** 25), False), (F(5, 4), F(1, 2 ** 24), True),
              (F(7, 4), F(1, 2 ** 24), False), (F(5, 2), F(1, 2 ** 23), True), (F(7, 2), F(1, 2 ** 23), False),
              (F(5), F(1, 2 ** 22), True)]


def _code_by_fma_rule(v: float, s: F) -> int:
    a = abs(F(v))
    passed_not = 0  # midpoints fl32(|v| / s) has not passed
    for t, h, le in _MIDPOINTS:
        d = _round_f32(a - t * s)  # one rounding, as an fma
        passed_not += (d <= h * s) if le else (d < -h * s)
    c = 7 - passed_not
    return c | 8 if c and v < 0 else c


def _e4m3_positive() -> list:
    vals = []
    for e in range(16):
        for m in range(8):
            if e == 15 and m == 7:  # NaN
                continue
            v = F(m, 8) * F(2) ** -6 if e == 0 else (1 + F(m, 8)) * F(2) ** (e - 7)
            if v > 0:
                vals.append(v)
    return vals


def test_midpoint_spacings_are_half_ulps():
    """h is half the gap to t's fp32 neighbour on the side the rule looks at: above t for a "<=" midpoint
    (0.25 is a power of two, so only that side's gap applies), below t for a "<" one."""
    for t, h, le in _MIDPOINTS:
        t32 = np.float32(float(t))
        if le:
            assert F(float(np.nextafter(t32, np.float32(np.inf)))) - t == 2 * h
        else:
            assert t - F(float(np.nextafter(t32, np.float32(0)))) == 2 * h
        # every midpoint's last mantissa bit is even, so a quotient halfway to a neighbour rounds onto t
        assert int(np.array(t32).view(np.uint32)) & 1 == 0


@pytest.mark.parametrize("sign", [1, -1])
def test_fma_rule_matches_rounded_quotient_for_every_e4m3_scale(sign):
    rng = np.random.default_rng(7)
    n = bad = 0
    for s in _e4m3_positive():
        for t, _, _ in _MIDPOINTS:
            for mult in (1.0, 1 + 2.0 ** -24, 1 - 2.0 ** -24, 1 + 2.0 ** -23, 1 - 2.0 ** -23):
                c0 = np.float32(float(t * s) * mult)
                vs = [c0]
                up = down = c0
                for _ in range(3):
                    up = np.nextafter(up, np.float32(np.inf))
                    down = np.nextafter(down, np.float32(0))
                    vs += [up, down]
                for v in vs:
                    v = float(np.float32(sign * v))
                    n += 1
                    bad += _code_by_fma_rule(v, s) != _code_of_quotient(v, s)
        for v in rng.uniform(-8, 8, 20) * float(s):
            v = float(np.float32(sign * abs(v)))
            n += 1
            bad += _code_by_fma_rule(v, s) != _code_of_quotient(v, s)
    assert n > 30000 and bad == 0


def test_zero_and_extremes():
    for s in (F(1, 512), F(1), F(448)):
        assert _code_by_fma_rule(0.0, s) == _code_of_quotient(0.0, s) == 0
        assert _code_by_fma_rule(-0.0, s) == 0
        assert _code_by_fma_rule(3.0e38, s) == 7 and _code_by_fma_rule(-3.0e38, s) == 15
