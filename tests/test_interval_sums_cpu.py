"""The lemma behind the pool and gather kernels' fast path, checked with exact rational arithmetic (no GPU).

The kernels sum a pooled entry's bf16 values twice in fp32, in the definition's tree order (p children left to
right at every level), every addition rounded toward +inf in one copy and toward -inf in the other.  They use the
common value when both copies agree and the scaled value sum * 2^-(l log2 p) is zero or a normal fp32 number, and
round that to bf16.  The claim is that the result is then exactly the oracle's pooled value (fp64 tree sum, one bf16
rounding of sum / p^l).  Here fp32 directed rounding is emulated exactly (fractions and float32 neighbours), on
adversarial bf16 inputs: zeros of both signs, subnormals, exponents spread over 2^-140 .. 2^20."""

from __future__ import annotations

from fractions import Fraction

import numpy as np
import pytest

from oracle import lighthouse as O

INF32 = np.float32(np.inf)


def _round_up(q: Fraction) -> np.float32:
    """The smallest float32 >= q (q finite and within the float32 range)."""
    c = np.float32(float(q))
    while Fraction(float(c)) < q:
        c = np.nextafter(c, INF32)
    while Fraction(float(np.nextafter(c, -INF32))) >= q:
        c = np.nextafter(c, -INF32)
    return c


def _round_down(q: Fraction) -> np.float32:
    return -_round_up(-q)


def _add_up(a: np.float32, b: np.float32) -> np.float32:
    s = Fraction(float(a)) + Fraction(float(b))
    r = _round_up(s)
    if s == 0:  # exact zero: +0 under upward rounding unless both operands are -0
        r = np.float32(-0.0) if (np.signbit(a) and np.signbit(b)) else np.float32(0.0)
    return r


def _add_down(a: np.float32, b: np.float32) -> np.float32:
    s = Fraction(float(a)) + Fraction(float(b))
    r = _round_down(s)
    if s == 0:  # exact zero: -0 under downward rounding unless both operands are +0
        r = np.float32(0.0) if (not np.signbit(a) and not np.signbit(b)) else np.float32(-0.0)
    return r


def _tree(values, p, lev, add):
    """Sum of p^lev values in the definition's order with the given addition."""
    if lev == 0:
        return values[0]
    w = p ** (lev - 1)
    acc = None
    for c in range(p):
        child = _tree(values[c * w:(c + 1) * w], p, lev - 1, add)
        acc = child if acc is None else add(acc, child)
    return acc


def _f64_add(a, b):
    return a + b  # Python floats: IEEE binary64, round to nearest even


def _hard_bf16(rng, n):
    """bf16 values (as float64): random sign and 7-bit fraction, exponents per entry in a band or spread wide,
    about one in eight a zero of either sign."""
    sign = rng.choice([-1.0, 1.0], n)
    mant = 1 + rng.integers(0, 128, n) / 128
    if rng.random() < 0.5:
        e = rng.integers(-140, 21, n)
    else:
        top = rng.integers(-138, 21)
        e = top - rng.integers(0, 3, n)
    x = sign * mant * np.exp2(e.astype(np.float64))
    x[rng.random(n) < 0.125] = 0.0
    x = sign * np.abs(O.bf16_round(x))  # bf16 values; keeps the sign of zeros
    return x


@pytest.mark.parametrize("p,lev", [(2, 1), (4, 1), (8, 1), (4, 2), (2, 3), (4, 3)])
def test_closed_interval_gives_the_oracles_pooled_value(p, lev):
    rng = np.random.default_rng(1000 * p + lev)
    closed = open_ = 0
    for _ in range(120 if p ** lev <= 16 else 30):
        vals = _hard_bf16(rng, p ** lev)
        v32 = [np.float32(v) for v in vals]  # exact: bf16 values are float32 values
        up = _tree(v32, p, lev, _add_up)
        dn = _tree(v32, p, lev, _add_down)
        exact = sum(Fraction(float(v)) for v in vals)
        # the bracket always holds
        assert Fraction(float(dn)) <= exact <= Fraction(float(up))
        s64 = _tree(list(vals), p, lev, _f64_add)
        want = O.bf16_round(np.float64(s64) / float(p ** lev))
        if np.float32(up) != np.float32(dn) and not (up == 0 and dn == 0):
            open_ += 1
            continue
        closed += 1
        # both copies agree: every partial sum was exact, so the fp64 tree gives the same value
        assert Fraction(float(up)) == exact and Fraction(s64) == exact
        scaled = np.float32(float(up) / float(p ** lev))  # exact power-of-two scaling while normal or zero
        if scaled != 0 and abs(scaled) < np.finfo(np.float32).tiny:
            continue  # subnormal: the kernels take the fp64 route here
        got = O.bf16_round(np.float64(scaled))
        assert O.bf16_bits(got) == O.bf16_bits(want), (vals, up, got, want)
    assert closed > 0 and open_ > 0  # both branches were exercised
