"""Independent exact/textbook helpers used to pin the oracle.

Nothing here imports the oracle.  Rounding is done in exact rational arithmetic (``fractions.Fraction``) and
attention by plain Python loops, so a mistake in the oracle's numpy code cannot be mirrored here by construction.
"""

from __future__ import annotations

import math
import struct
from fractions import Fraction


def round_fraction(x: Fraction, sig_bits: int, min_exp: int, max_exp: int) -> Fraction | float:
    """Nearest binary floating-point value to ``x`` with ``sig_bits`` significant bits, ties to even.

    ``min_exp`` is the smallest normal binade (subnormals share its quantum); magnitudes that round to
    ``2**(max_exp+1)`` or beyond give ``±inf``."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, min_exp)
    quantum = Fraction(2) ** (e - (sig_bits - 1))
    y = a / quantum
    n = y.numerator // y.denominator
    rem = y - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    r = n * quantum
    if r >= Fraction(2) ** (max_exp + 1):
        return sign * math.inf
    return sign * r


def to_bf16_exact(x) -> float:
    r = round_fraction(Fraction(x), 8, -126, 127)
    return float(r)


def to_fp32_exact(x) -> float:
    r = round_fraction(Fraction(x), 24, -126, 127)
    return float(r)


def bf16_value_of_bits(b: int) -> float:
    return struct.unpack("<f", struct.pack("<I", (b & 0xFFFF) << 16))[0]


def textbook_causal_attention(q, k, v):
    """Row-by-row causal softmax attention with plain Python loops (lists of lists of floats)."""
    S = len(q)
    d = len(q[0])
    scale = 1.0 / math.sqrt(d)
    out = []
    for a in range(S):
        logits = [sum(q[a][i] * k[b][i] for i in range(d)) * scale for b in range(a + 1)]
        mx = max(logits)
        w = [math.exp(x - mx) for x in logits]
        z = sum(w)
        out.append([sum(w[b] * v[b][i] for b in range(a + 1)) / z for i in range(d)])
    return out
