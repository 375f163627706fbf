"""Exhaustive-search restatements used to pin the oracle.

These do not call the oracle and share nothing with it: the quantiser here
searches every scale exponent and every code instead of computing them.

Arithmetic is exact: values are binary32 numbers held as Python floats
(binary64), steps are powers of two, and every difference |v - k*2^e| taken
here spans fewer than 30 significant bits, so binary64 represents it exactly.
"""
from __future__ import annotations

import math
from fractions import Fraction

CODE_MIN, CODE_MAX = -7, 7
E_MIN, E_MAX = -127, 126


def bf_quantize(values) -> tuple[int, list[int]]:
    """Scale byte and codes of one group by exhaustive search.

    Walk every exponent from the smallest up and take the first one at which no
    value falls outside the code range [-7, 7] * 2^e; then, per value, try every
    code and keep the nearest, preferring the even code on a tie.
    """
    vals = [float(v) for v in values]
    for e in range(E_MIN, E_MAX + 1):
        step = math.ldexp(1.0, e)
        if all(CODE_MIN * step <= v <= CODE_MAX * step for v in vals):
            codes = []
            for v in vals:
                best_k, best_d = None, None
                for k in range(CODE_MIN, CODE_MAX + 1):
                    d = abs(v - k * step)
                    if best_d is None or d < best_d or (d == best_d and k % 2 == 0):
                        best_k, best_d = k, d
                codes.append(best_k)
            return e + 127, codes
    raise ValueError("no exponent in range fits the group")


def value_of(code: int, byte: int) -> Fraction:
    """Exact value of a code under a scale byte."""
    return code * Fraction(2) ** (byte - 127)
