"""The codec's device shortcuts, modelled on the CPU and held against the
oracle's rounding (no GPU needed).

The kernels do not compute a scale or a code the way the oracle does (a
search over e or over binary16 values, rounding in binary64). They take
shortcuts whose exactness rests on an argument, written beside them in
``echo_codec.cuh``:

* power-of-two scale: the byte is read from the exponent and mantissa fields
  of the maximum, and the code is one fused fma(v, 2^-e, 1.5 * 2^23);

* scale: u = A * RU(1/7), rounded up, then rounded up again to binary16, is
  never below the answer and at most one binary16 step above it, so one exact
  test of the step below settles it;
* code: z = RN(v * inv + kZ) keeps the code in byte 2 and a 16-bit fraction
  below it; when that fraction is at least kZMargin units of 2^-16 from a
  midpoint, the code is the exact nearest one, whatever error up to 2^-23
  the reciprocal estimate inv carries;
* code of a value with 8 significant bits (a bf16 partial that carries no
  correction): the nearest code unless the fraction is below kZTie, which
  only an exact midpoint reaches, and then an odd code moves down by one.

This test restates them in binary64 and long double, with the constants read
from the header, and checks them against the oracle on groups with ties,
near-ties, bf16 partials, subnormals and wide ranges. It reads the header as
text only; nothing of the CUDA path runs.
"""
from __future__ import annotations

import os
import re

import numpy as np
import pytest

from bit_error_compensated_rank_b200.workloads import bf16_bits, bf16_to_f32, outlier_gaussian
from oracle.oracle import FP16_SCALE
from pins import _many_random_groups, _quantise_rows_with_oracle

# v * inv + kZ rounded once to binary32 needs about 56 significant bits before
# the rounding: x86 long double (64) holds it, binary64 (53) does not.
pytestmark = pytest.mark.skipif(np.finfo(np.longdouble).nmant < 60,
                                reason="needs a long double with at least 60 significand bits")

CODEC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                     "bit_error_compensated_rank_b200", "csrc", "echo_codec.cuh")
G = 32


def _constants():
    text = open(CODEC).read()
    kz = float(re.search(r"constexpr float kZ = ([0-9.]+)f;", text).group(1))
    margin = int(re.search(r"constexpr uint32_t kZMargin = (\d+);", text).group(1))
    seventh = int(re.search(r"__fmul_ru\(A, __uint_as_float\((0x[0-9A-Fa-f]+)u\)\)", text).group(1), 16)
    return np.float32(kz), margin, np.uint32(seventh).view(np.float32)


def _ru32(x: np.ndarray) -> np.ndarray:
    """Exact binary64 values rounded up to binary32."""
    f = x.astype(np.float32)
    lo = f.astype(np.float64) < x
    f[lo] = np.nextafter(f[lo], np.float32(np.inf))
    return f


def _ru16(x: np.ndarray) -> np.ndarray:
    """binary32 values rounded up to binary16 (beyond 65504: infinity)."""
    with np.errstate(over="ignore"):
        h = x.astype(np.float16)
        lo = h.astype(np.float64) < x.astype(np.float64)
        h[lo] = np.nextafter(h[lo], np.float16(np.inf))
    return h


def _device_scale(A: np.ndarray, seventh: np.float32) -> np.ndarray:
    u = _ru32(A.astype(np.float64) * np.float64(seventh))  # the product is exact in binary64
    h = np.minimum(_ru16(u).view(np.uint16).astype(np.int64), 0x7BFF)
    below = np.maximum(h - 1, 0).astype(np.uint16).view(np.float16).astype(np.float64)
    down = (h > 1) & (7.0 * below >= A.astype(np.float64))
    return h - down


def _device_codes(v: np.ndarray, h: np.ndarray, kz: np.float32, margin: int, eta: float):
    """z-form codes of rows v under binary16 steps h, with the reciprocal off
    by the relative error eta; returns (codes, lane flagged for the exact path)."""
    s = h.astype(np.uint16).view(np.float16).astype(np.float32)
    inv = np.where(s > 0, np.float32(1) / np.where(s > 0, s, 1), 0).astype(np.float64) * (1 + eta)
    z = (v.astype(np.longdouble) * inv[:, None].astype(np.longdouble) + np.longdouble(kz)).astype(np.float32)
    bits = z.view(np.uint32).astype(np.int64)
    codes = (bits >> 16) - 0x4340
    flagged = ((bits & 0xFFFF) < margin).reshape(v.shape[0], -1, 8).any(axis=2)  # per lane of 8
    return codes, np.repeat(flagged, 8, axis=1)


def _zbits(v: np.ndarray, h: np.ndarray, kz: np.float32, eta: float) -> np.ndarray:
    """Bit patterns of z = RN(v * inv + kZ) for rows v under binary16 steps h,
    the reciprocal off by the relative error eta."""
    s = h.astype(np.uint16).view(np.float16).astype(np.float32)
    inv = np.where(s > 0, np.float32(1) / np.where(s > 0, s, 1), 0).astype(np.float64) * (1 + eta)
    z = (v.astype(np.longdouble) * inv[:, None].astype(np.longdouble) + np.longdouble(kz)).astype(np.float32)
    return z.view(np.uint32).astype(np.int64)


def _bf16_rows():
    """Rows of bf16 values below saturation: the benchmark's partials, bf16
    roundings of wide-range groups, rows of exact midpoints (k + 1/2) * s of
    few-bit binary16 steps s, and the bf16 values nearest to the midpoints of
    random binary16 steps (each an exact tie or a near one)."""
    partials = bf16_to_f32(outlier_gaussian(1, (1 << 15) * G, seed=5, call=0)).reshape(-1, G)
    mixed = np.clip(_many_random_groups(1 << 14, G, seed=19), -4e5, 4e5).astype(np.float32)
    mixed = bf16_to_f32(bf16_bits(mixed))
    g = np.random.default_rng(21)
    rows = 1 << 14
    m = g.integers(1, 16, (rows, 1))
    q = g.integers(-24, 13, (rows, 1))
    s = m * np.exp2(q.astype(np.float64))          # a binary16 value: 4 bits, 2^-24 .. 61440
    k = g.integers(-7, 7, (rows, G)) + 0.5          # midpoints -6.5 .. 6.5: 8 bits or fewer
    mid = k * s
    mid[:, 0] = 7 * s[:, 0]                         # the maximum makes s the group's step
    hs = g.integers(0x0001, 0x7800, (rows, 1)).astype(np.uint16).view(np.float16).astype(np.float64)
    near = (g.integers(-7, 7, (rows, G)) + 0.5) * hs
    near[:, 0] = 7 * hs[:, 0]
    near = bf16_to_f32(bf16_bits(near.astype(np.float32)))
    out = np.concatenate([partials, mixed, mid.astype(np.float32), near]).astype(np.float32)
    assert np.array_equal(bf16_to_f32(bf16_bits(out)), out)  # every value is a bf16
    return out


def _rows():
    mixed = _many_random_groups(1 << 15, G, seed=9)
    mixed = np.clip(mixed, -4e5, 4e5).astype(np.float32)  # below saturation (7 * 65504)
    partials = bf16_to_f32(outlier_gaussian(1, (1 << 15) * G, seed=3, call=0)).reshape(-1, G)
    g = np.random.default_rng(11)  # near ties: a few binary32 ulps around (k + 1/2) * s
    hs = g.integers(0x0400, 0x7000, (1 << 14, 1)).astype(np.uint16).view(np.float16).astype(np.float64)
    k = g.integers(-7, 7, (1 << 14, G)) + 0.5
    k[:, 0] = 7
    near = (k * hs).astype(np.float32)
    off = g.integers(-3, 4, near.shape).astype(np.int32)
    off[:, 0] = 0
    near = (near.view(np.int32) + off).view(np.float32)
    return np.concatenate([mixed, partials, near]).astype(np.float32)


def test_binary16_scale_one_test_rule(oracle):
    _, _, seventh = _constants()
    x = _rows()
    h_oracle, _ = _quantise_rows_with_oracle(oracle, x, G, FP16_SCALE)
    A = np.abs(x).max(axis=1)
    assert np.array_equal(_device_scale(A, seventh), h_oracle)
    # every boundary 7*s of the rule and a few ulps either side
    s = np.arange(1, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)
    b = (7.0 * s).astype(np.float32)
    for d in range(-2, 3):
        Ab = (b.view(np.int32) + d).view(np.float32)
        rows = np.zeros((Ab.size, G), np.float32)
        rows[:, 0] = Ab
        h_b, _ = _quantise_rows_with_oracle(oracle, rows, G, FP16_SCALE)
        assert np.array_equal(_device_scale(Ab, seventh), h_b), d


def test_binary16_zform_codes_exact_when_not_flagged(oracle):
    kz, margin, _ = _constants()
    assert kz.view(np.uint32) == 0x43408002 and margin >= 1
    x = _rows()
    h, q = _quantise_rows_with_oracle(oracle, x, G, FP16_SCALE)
    for eta in (0.0, 2.0 ** -23, -(2.0 ** -23)):
        codes, flagged = _device_codes(x, h, kz, margin, eta)
        wrong = codes != q
        assert not (wrong & ~flagged).any(), (eta, np.argwhere(wrong & ~flagged)[:4])
        # exact ties are flagged, so the exact path sees every one of them
        s = h.astype(np.uint16).view(np.float16).astype(np.float64)
        ratio = x.astype(np.float64) / np.where(s > 0, s, 1)[:, None]
        ties = (s[:, None] > 0) & (ratio - np.floor(ratio) == 0.5)
        assert ties.any() and flagged[ties].all()
    # bf16 partials hold exact ties often enough to matter for the kernel's cost
    assert ties.mean() > 1e-4


def test_binary16_codes_of_bf16_values_settle_ties_without_the_exact_path(oracle):
    """Values of 8 significant bits: the fast code, with an odd code moved
    down by one where the fraction is below kZTie (exact midpoints only), is
    the oracle's nearest code for every value, whatever reciprocal error up
    to 2^-23; and no value other than an exact midpoint reaches kZTie."""
    kz, margin, _ = _constants()
    tie_bound = int(re.search(r"constexpr uint32_t kZTie = (\d+);", open(CODEC).read()).group(1))
    x = _bf16_rows()
    h, q = _quantise_rows_with_oracle(oracle, x, G, FP16_SCALE)
    assert (h < 0x7BFF).all()  # no saturated group: those take the exact path
    s = h.astype(np.uint16).view(np.float16).astype(np.float64)
    ratio = x.astype(np.float64) / np.where(s > 0, s, 1)[:, None]
    ties = (s[:, None] > 0) & (ratio - np.floor(ratio) == 0.5)
    assert ties.sum() > 10000
    for eta in (0.0, 2.0 ** -23, -(2.0 ** -23)):
        bits = _zbits(x, h, kz, eta)
        codes = (bits >> 16) - 0x4340
        low = bits & 0xFFFF
        assert np.array_equal(low < tie_bound, ties), eta
        fixed = codes - ((low < tie_bound) & (codes % 2 != 0))
        assert np.array_equal(fixed, q), (eta, np.argwhere(fixed != q)[:4])


def _device_scale_byte(A: np.ndarray) -> np.ndarray:
    """The kernels' closed form: byte = max(0, E - 2 + [M > 0x600000])."""
    u = A.astype(np.float32).view(np.uint32).astype(np.int64)
    b = (u >> 23) - 2 + ((u & 0x7FFFFF) > 0x600000)
    return np.maximum(b, 0)


def test_power_of_two_scale_closed_form_and_fused_codes(oracle):
    """Default format: the scale byte read from the bits of the maximum, and
    the code from one fused fma(v, 2^-e, 1.5 * 2^23), against the oracle's
    search over e and its binary64 rounding."""
    x = _rows()
    # every exponent field up to the oracle's domain (|x| < 2^120), mantissas
    # around the 7/4 boundary
    g = np.random.default_rng(12)
    E = np.repeat(np.arange(0, 246), 16)
    M = np.clip(0x600000 + g.integers(-3, 4, E.size), 0, 0x7FFFFF)
    A = ((E << 23) | M).astype(np.uint32).view(np.float32)
    edge = np.zeros((A.size, G), np.float32)
    edge[:, 0] = A
    edge[:, 1:] = A[:, None] * g.uniform(-1, 1, (A.size, G - 1)).astype(np.float32)
    x = np.concatenate([x, edge])
    b_oracle, q_oracle = _quantise_rows_with_oracle(oracle, x, G, 0)
    b = _device_scale_byte(np.abs(x).max(axis=1))
    assert np.array_equal(b, b_oracle)
    inv = np.ldexp(1.0, 127 - b)  # 2^-e, a normal binary32 for every byte the rule gives
    t = (x.astype(np.longdouble) * inv[:, None].astype(np.longdouble) + np.longdouble(1.5 * 2 ** 23)).astype(np.float32)
    codes = t.view(np.uint32).astype(np.int64) - 0x4B400000
    assert np.array_equal(codes, q_oracle)
