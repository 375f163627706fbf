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


# ---- binary16-scale variant ------------------------------------------------
def _half_table():
    """Every positive finite binary16 value in increasing order, decoded by
    numpy (not by the oracle), with its bit pattern."""
    import numpy as np
    bits = np.arange(1, 0x7C00, dtype=np.uint16)
    return bits, bits.view(np.float16).astype(np.float64)


def bf_quantize_f16(values) -> tuple[int, list[int]]:
    """Binary16 scale pattern and codes of one group by exhaustive search.

    The scale is the first positive finite binary16, in increasing order, whose
    7-fold covers the largest magnitude (the largest finite one, 65504, when
    none does; 0 for an all-zero group). Every code in [-7, 7] is tried per
    value with exact rational distances; a tie goes to the even code.
    """
    import numpy as np
    vals = [Fraction(float(v)) for v in values]
    A = max(abs(v) for v in vals)
    if A == 0:
        return 0, [0] * len(vals)
    bits, table = _half_table()
    ok = np.flatnonzero(7 * table >= float(A))  # 7*s and A are exact in binary64
    i = int(ok[0]) if ok.size else len(table) - 1
    h, s = int(bits[i]), Fraction(float(table[i]))
    codes = []
    for v in vals:
        best_k, best_d = None, None
        for k in range(CODE_MIN, CODE_MAX + 1):
            d = abs(v - k * s)
            if best_d is None or d < best_d or (d == best_d and k % 2 == 0):
                best_k, best_d = k, d
        codes.append(best_k)
    return h, codes


def half_fraction(h: int) -> Fraction:
    """Exact value of a binary16 bit pattern, decoded by numpy."""
    import numpy as np
    return Fraction(float(np.array([h], dtype=np.uint16).view(np.float16)[0]))


def bf16_round_bits(x: float) -> float:
    """Nearest bf16 to a binary32 value, ties to even, by integer arithmetic on
    the bit pattern: add 0x7FFF plus the lowest kept bit, drop the low half."""
    import struct
    u = struct.unpack("<I", struct.pack("<f", x))[0]
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return struct.unpack("<f", struct.pack("<I", u))[0]


# ---- vectorised versions for many random groups -----------------------------
def bf_quantize_many(v):
    """Scale bytes and codes of many groups (rows of v, binary32 values) by
    the same search, vectorised: the exponent is the first e >= -127 with
    every |v| <= 7*2^e (found from an estimate and settled by exact tests on
    both sides), and each code is the k in [-7, 7] at the least distance
    |v - k*2^e|, a tie going to the even k. Everything is exact in binary64."""
    import numpy as np
    x = np.asarray(v, dtype=np.float64)
    A = np.abs(x).max(axis=1)
    e = np.full(A.shape, -127, dtype=np.int64)
    nz = A > 0
    _, ex = np.frexp(A[nz] / 7.0)
    e[nz] = np.maximum(ex - 1, -127)
    for _ in range(3):  # settle: smallest e with A <= 7*2^e
        up = A > 7.0 * np.ldexp(1.0, e)
        e = np.where(up, e + 1, e)
        down = (e > -127) & (A <= 7.0 * np.ldexp(1.0, e - 1))
        e = np.where(down, e - 1, e)
    step = np.ldexp(1.0, e)[:, None]
    best_k = np.zeros(x.shape, dtype=np.int64)
    best_d = np.full(x.shape, np.inf)
    for k in range(CODE_MIN, CODE_MAX + 1):
        d = np.abs(x - k * step)
        better = (d < best_d) | ((d == best_d) & (k % 2 == 0))
        best_k = np.where(better, k, best_k)
        best_d = np.where(better, d, best_d)
    return (e + 127).astype(np.int64), best_k


def bf_quantize_f16_many(v):
    """The binary16-scale quantiser for many groups: the scale is the first
    binary16 (numpy's table) whose 7-fold covers the group's maximum, found
    by a search over the sorted table (65504 past it, 0 for a zero group);
    codes as in bf_quantize_many."""
    import numpy as np
    x = np.asarray(v, dtype=np.float64)
    A = np.abs(x).max(axis=1)
    bits, table = _half_table()
    i = np.searchsorted(7.0 * table, A, side="left")  # first index with 7*s >= A
    i = np.minimum(i, len(table) - 1)
    h = np.where(A == 0, 0, bits[i].astype(np.int64))
    s = np.where(A == 0, 0.0, table[i])[:, None]
    best_k = np.zeros(x.shape, dtype=np.int64)
    best_d = np.full(x.shape, np.inf)
    for k in range(CODE_MIN, CODE_MAX + 1):
        d = np.abs(x - k * s)
        better = (d < best_d) | ((d == best_d) & (k % 2 == 0))
        best_k = np.where(better, k, best_k)
        best_d = np.where(better, d, best_d)
    return h, np.where((A == 0)[:, None], 0, best_k)  # a zero group has no step: codes 0
