"""Plant plausible mistakes in copies of the oracle and require the pins to
catch every one.

Each mutant is the oracle's C source with one textual change, compiled to a
temporary library on the CPU. A mutant passes this test only if at least one
pin in ``pins.ALL_PINS`` fails on it; a mutant no pin notices would mean the
pins do not actually tie that part of the oracle down.
"""
import os
import shutil
import subprocess

import pytest

from oracle.oracle import Oracle
from pins import ALL_PINS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE_DIR = os.path.join(ROOT, "oracle")

MUTANTS = [
    ("ties_away_from_zero",
     "double t = nearbyint(ldexp((double)v[k], -e));",
     "double t = round(ldexp((double)v[k], -e));"),
    ("scale_strict_boundary",
     "while (!(A <= ldexp(7.0, e))) {",
     "while (!(A < ldexp(7.0, e))) {"),
    ("scale_range_8",
     "while (!(A <= ldexp(7.0, e))) {",
     "while (!(A <= ldexp(8.0, e))) {"),
    ("absmax_wrong_compare",
     "if (a > A)\n            A = a;",
     "if (a < A)\n            A = a;"),
    ("nibbles_swapped",
     "out[j] = (uint8_t)(lo | (hi << 4));",
     "out[j] = (uint8_t)(hi | (lo << 4));"),
    ("dequant_off_by_one",
     "return (float)ldexp((double)q, b - 127);",
     "return (float)ldexp((double)q, b - 126);"),
    ("sum_skips_rank0",
     "for (int r = 0; r < P; r++) {\n                float d",
     "for (int r = 1; r < P; r++) {\n                float d"),
    ("sum_reversed_order",
     "float d = restore(q1[(size_t)r * m + i], b1[(size_t)r * ngroups + g], half_scale);",
     "float d = restore(q1[(size_t)(P - 1 - r) * m + i], b1[(size_t)(P - 1 - r) * ngroups + g], half_scale);"),
    ("sum_in_binary64",
     "float sum = 0.0f;",
     "double sum = 0.0;"),
    ("error_sign_flipped",
     "float err = S[k] - Y;",
     "float err = Y - S[k];"),
    ("combine_minus",
     "c[i] = from_fast + from_slow;",
     "c[i] = from_fast - from_slow;"),
    ("lambda_on_slow",
     "float from_fast = lambda * f[i];",
     "float from_fast = lambda * s[i];"),
    ("every_rank_injects",
     "if (enable && !owner_sum && owner[g] == r)",
     "if (enable && !owner_sum)"),
    ("wrong_owner",
     "owner[g] = (int32_t)((g * (size_t)G) / seg);",
     "owner[g] = (int32_t)(((g * (size_t)G) / seg + 1) % (size_t)P);"),
    ("fast_uses_slow_beta",
     "float f_keep = beta_f * f[i];",
     "float f_keep = beta_s * f[i];"),
    ("slow_weights_swapped",
     "float s_new = one_minus_beta_s * err;",
     "float s_new = beta_s * err;"),
    ("state_not_updated",
     "f[i] = f_keep + f_new;",
     "f[i] = f[i];"),
    ("captures_stage1_error_instead",
     "float Y = restore(Q[i], bq, half_scale);",
     "float Y = S[k];"),
    ("correction_not_added",
     "v[k] = u + c[i];",
     "v[k] = u;"),
    # operation order: a product fused into the following add, or the adds
    # regrouped (each is the same real-number expression, rounded differently)
    ("combine_fma",
     "c[i] = from_fast + from_slow;",
     "c[i] = fmaf(lambda, f[i], from_slow);"),
    ("combine_fma_slow",
     "c[i] = from_fast + from_slow;",
     "c[i] = fmaf(one_minus_lambda, s[i], from_fast);"),
    ("combine_increment",
     "c[i] = from_fast + from_slow;",
     "c[i] = s[i] + lambda * (f[i] - s[i]);"),
    ("ema_fast_fma",
     "f[i] = f_keep + f_new;",
     "f[i] = fmaf(beta_f, f[i], f_new);"),
    ("ema_fast_fma_new",
     "f[i] = f_keep + f_new;",
     "f[i] = fmaf(one_minus_beta_f, err, f_keep);"),
    ("ema_fast_increment",
     "f[i] = f_keep + f_new;",
     "f[i] = f[i] + one_minus_beta_f * (err - f[i]);"),
    ("ema_slow_fma",
     "s[i] = s_keep + s_new;",
     "s[i] = fmaf(beta_s, s[i], s_new);"),
    ("ema_slow_fma_new",
     "s[i] = s_keep + s_new;",
     "s[i] = fmaf(one_minus_beta_s, err, s_keep);"),
    ("ema_slow_increment",
     "s[i] = s_keep + s_new;",
     "s[i] = s[i] + one_minus_beta_s * (err - s[i]);"),
    ("sender_reassoc",
     "v[k] = u + c[i];",
     "v[k] = sender_ef ? xi + (eps[(size_t)r * m + i] + c[i]) : u + c[i];"),
    ("sender_correction_first",
     "v[k] = u + c[i];",
     "v[k] = sender_ef ? (xi + c[i]) + eps[(size_t)r * m + i] : u + c[i];"),
    # variants
    ("sender_error_not_kept",
     "eps[(size_t)r * m + i] = v[k] - restored;",
     "eps[(size_t)r * m + i] = 0.0f;"),
    ("sender_error_sign_flipped",
     "eps[(size_t)r * m + i] = v[k] - restored;",
     "eps[(size_t)r * m + i] = restored - v[k];"),
    ("sender_error_not_added",
     "u = xi + eps[(size_t)r * m + i];",
     "u = xi;"),
    ("sender_error_wrong_rank",
     "u = xi + eps[(size_t)r * m + i];",
     "u = xi + eps[(size_t)((r + 1) % P) * m + i];"),
    ("owner_sum_adds_twice",
     "sum = sum + c[i];",
     "sum = sum + c[i] + c[i];"),
    ("owner_sum_sender_also_adds",
     "if (enable && !owner_sum && owner[g] == r)",
     "if (enable && owner[g] == r)"),
    ("owner_sum_starts_from_correction",
     [("float sum = 0.0f;", "float sum = (enable && owner_sum) ? c[i] : 0.0f;"),
      ("if (enable && owner_sum)\n                sum = sum + c[i];", "")]),
    # binary16-scale variant
    ("f16_scale_strict_boundary",
     "if (7.0 * echo_oracle_half_value(mid) >= A)",
     "if (7.0 * echo_oracle_half_value(mid) > A)"),
    ("f16_scale_range_8",
     "if (7.0 * echo_oracle_half_value(mid) >= A)",
     "if (8.0 * echo_oracle_half_value(mid) >= A)"),
    ("f16_saturates_to_infinity",
     "if (7.0 * echo_oracle_half_value(hi) < A)\n        return hi;",
     "if (7.0 * echo_oracle_half_value(hi) < A)\n        return 0x7C00;"),
    ("f16_ties_to_odd",
     "(k + 0.5) * s && (k % 2) == 1)",
     "(k + 0.5) * s && (k % 2) == 0)"),
    ("f16_ties_away_from_zero",
     "(k + 0.5) * s && (k % 2) == 1)",
     "(k + 0.5) * s)"),
    ("f16_codes_truncated",
     "while (k < 7 && a > (k + 0.5) * s)",
     "while (k < 7 && a >= (k + 1) * s)"),
    ("f16_subnormal_scale_decoded_wrong",
     "ldexp((double)frac, -24)",
     "ldexp((double)frac, -25)"),
    ("f16_bf16_output_ties_up",
     "r = (fmod(lo / step, 2.0) == 0.0) ? lo : hi;",
     "r = hi;"),
    ("f16_error_against_unrounded_output",
     [("Y = echo_oracle_round_bf16(Y);", ";"),
      ("int so = store_output(out, dtype, i, Y);",
       "int so = store_output(out, dtype, i, (half_scale && dtype == ECHO_ORACLE_BF16) ? "
       "echo_oracle_round_bf16(Y) : Y);")]),
    ("f16_wire_big_endian",
     "out[2 * t] = (uint8_t)(scale & 0xFF);\n        out[2 * t + 1] = (uint8_t)((scale >> 8) & 0xFF);",
     "out[2 * t + 1] = (uint8_t)(scale & 0xFF);\n        out[2 * t] = (uint8_t)((scale >> 8) & 0xFF);"),
]


@pytest.fixture(scope="module")
def mutant_dir(tmp_path_factory):
    return tmp_path_factory.mktemp("oracle_mutants")


def _edits(entry):
    """A mutant is (name, old, new) or (name, [(old, new), ...])."""
    if len(entry) == 3:
        return [(entry[1], entry[2])]
    return entry[1]


@pytest.mark.parametrize("entry", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(mutant_dir, entry):
    name = entry[0]
    src = open(os.path.join(ORACLE_DIR, "echo_oracle.c")).read()
    for old, new in _edits(entry):
        assert src.count(old) == 1, f"mutation site for {name} not unique/present: {old!r}"
        src = src.replace(old, new)
    work = os.path.join(str(mutant_dir), name)
    os.makedirs(work, exist_ok=True)
    shutil.copy(os.path.join(ORACLE_DIR, "echo_oracle.h"), work)
    with open(os.path.join(work, "echo_oracle.c"), "w") as fh:
        fh.write(src)
    lib = os.path.join(work, "libmutant.so")
    subprocess.run(["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fPIC", "-shared",
                    "-o", lib, os.path.join(work, "echo_oracle.c"), "-lm"], check=True)
    orc = Oracle(lib)
    caught = None
    for pin in ALL_PINS:  # in order, cheapest first: the first failure is enough
        try:
            pin(orc)
        except Exception:  # any failure, assertion or error, counts as caught
            caught = pin.__name__
            break
    assert caught, f"no pin catches mutant {name}"
