"""Pins: checks that tie the CPU oracle to what the pages and the mathematics
fix, without trusting the oracle's own code.

Each pin takes an ``Oracle`` and raises ``AssertionError`` (or any error) when
the oracle disagrees. ``test_oracle_pins.py`` runs them on the oracle;
``test_oracle_mutants.py`` runs them on deliberately altered copies of it and
requires every alteration to be caught by at least one pin.

What the pages fix (Echo digests: [rit.work "Echo 4-bit GPU communication",
section "How Echo returns the error to later calls"], [heraldofai.com "Come
Echo permette ai modelli AI...", section "Come Echo evita che gli errori si
accumulino"]):
  * segments travel as 4-bit integers; the owner restores and sums them in high
    precision, then sends back a 4-bit total: at most two roundings per element
    whatever the group size;
  * the error of the owner's rounding is measured from the high-precision sum
    and added back in later calls, through a fast and a slow smoothed estimate;
  * with the correction, the running sum of injected error stays bounded;
    without it, it keeps growing.
Everything else (group, scale rule, rounding, op order, coefficients) is a
fixed reading, pinned here by hand-worked values and closed forms.
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np

from bit_error_compensated_rank_b200.workloads import bf16_bits, bf16_to_f32, gaussian, rng
from bruteforce import (bf16_round_bits, bf_quantize, bf_quantize_f16, bf_quantize_f16_many,
                        bf_quantize_many, half_fraction, value_of)
from oracle.oracle import FP16_SCALE, OWNER_SUM, SENDER_EF, Params

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
F32 = np.float32


def _load(name):
    with open(os.path.join(GOLDEN, name)) as fh:
        return json.load(fh)


def _parse_value(expr: str) -> np.float32:
    """Parse the small expressions of the boundary fixture: a decimal or a
    fraction, ``2^k``, ``a*2^k``, ``next_up(expr)``, ``FLT_MAX``."""
    expr = expr.strip()
    if expr == "FLT_MAX":
        return np.finfo(F32).max
    if expr.startswith("next_up(") and expr.endswith(")"):
        return np.nextafter(_parse_value(expr[len("next_up("):-1]), F32(np.inf))
    if "2^" in expr:
        coef, _, power = expr.partition("2^")
        coef = coef.rstrip("*") or "1"
        return F32(math.ldexp(float(Fraction(coef)), int(power)))
    return F32(float(Fraction(expr)))


def _frac_list(items):
    return [Fraction(t) for t in items]


def _values(x_bits_or_f32):
    a = np.asarray(x_bits_or_f32)
    return bf16_to_f32(a) if a.dtype == np.uint16 else a.astype(F32)


def _unpack_ref(packed) -> list[int]:
    """Layout reading: element 2j in the low nibble, 2j+1 in the high nibble,
    two's complement."""
    out = []
    for byte in np.asarray(packed, dtype=np.uint8).tolist():
        for nib in (byte & 0xF, byte >> 4):
            out.append(nib - 16 if nib >= 8 else nib)
    return out


# ---------------------------------------------------------------------------
# codec
# ---------------------------------------------------------------------------
def pin_scale_boundaries(orc):
    """Hand-worked scale bytes at every boundary of the scale rule, and halves
    rounded to even (fixture ``scale_boundaries.json``)."""
    fx = _load("scale_boundaries.json")
    for case in fx["scale_cases"]:
        A = _parse_value(case["A"])
        for sign in (1, -1):
            v = np.zeros(32, F32)
            v[5] = F32(sign) * A
            v[9] = A * F32(0.25)
            b, _ = orc.quantize_group(v)
            assert b == case["byte"], (case, b)
    t = fx["tie_cases_at_e0"]
    v = np.zeros(32, F32)
    vals = [F32(float(Fraction(s))) for s in t["values"]]
    v[:len(vals)] = vals
    b, q = orc.quantize_group(v)
    assert b == 127
    assert q[:len(vals)].tolist() == t["codes"], q[:len(vals)].tolist()


def _random_groups(count, G, seed):
    g = rng(seed, 99)
    groups = []
    for t in range(count):
        kind = t % 6
        if kind == 0:      # wide range of magnitudes
            v = g.standard_normal(G) * 2.0 ** g.integers(-140, 100)
        elif kind == 1:    # halves on a known grid: many ties
            e = int(g.integers(-120, 100))
            k = g.integers(-7, 7, G) + 0.5
            k[0] = 7 * (1 if g.random() < 0.5 else -1)
            v = k * 2.0 ** e
        elif kind == 2:    # subnormal binary32 values
            v = g.integers(-2 ** 20, 2 ** 20, G) * 2.0 ** -149
        elif kind == 3:    # a single non-zero value
            v = np.zeros(G)
            v[g.integers(0, G)] = g.standard_normal() * 2.0 ** g.integers(-30, 30)
        elif kind == 4:    # values near the 7*2^e boundary
            e = int(g.integers(-100, 100))
            v = g.uniform(-1, 1, G) * 7 * 2.0 ** e
            v[g.integers(0, G)] = np.nextafter(F32(7 * 2.0 ** e), F32(np.inf * (1 if g.random() < .5 else -1)))
        else:              # bf16-representable values
            v = bf16_to_f32(bf16_bits(g.standard_normal(G).astype(F32) * 3))
        groups.append(np.asarray(v, dtype=np.float64).astype(F32))
    return groups


def pin_quantizer_bruteforce(orc):
    """Scale byte and every code equal an exhaustive search over exponents and
    codes (ties to even), over ties, subnormals, boundaries and wide ranges."""
    for G in (32, 16, 64, 128, 8, 2):
        for v in _random_groups(60 if G == 32 else 24, G, seed=G):
            b, q = orc.quantize_group(v)
            bb, bq = bf_quantize(v.tolist())
            assert b == bb, (v, b, bb)
            assert q.tolist() == bq, (v, q.tolist(), bq)


def pin_roundtrip_bound(orc):
    """One rounding moves a value by at most half a step: |v - q*2^e| <= 2^(e-1)
    and |q| <= 7."""
    for v in _random_groups(120, 32, seed=7):
        b, q = orc.quantize_group(v)
        half = Fraction(2) ** (b - 127 - 1)
        for vi, qi in zip(v.tolist(), q.tolist()):
            assert -7 <= qi <= 7
            assert abs(Fraction(vi) - value_of(qi, b)) <= half


def pin_pack_layout(orc):
    """Two codes per byte, element 2j low, 2j+1 high, two's complement nibbles;
    unpack inverts pack for every pair of nibble values."""
    q = np.array([1, -1, -7, 7, 0, -2, 6, 3], np.int8)
    assert orc.pack(q).tolist() == [0xF1, 0x79, 0xE0, 0x36]
    pairs = [(a, b) for a in range(-8, 8) for b in range(-8, 8)]
    flat = np.array([c for p in pairs for c in p], np.int8)
    packed = orc.pack(flat)
    assert _unpack_ref(packed) == flat.tolist()
    assert orc.unpack(packed).tolist() == flat.tolist()
    for b in list(range(0, 253, 11)) + [253]:
        for qv in ((-3, -1, 0, 1, 3) if b == 253 else (-7, -1, 0, 3, 7)):
            assert Fraction(orc.dequant(qv, b)) == value_of(qv, b)


# ---------------------------------------------------------------------------
# whole calls
# ---------------------------------------------------------------------------
def _check_hand_fixture(orc, name, variant):
    fx = _load(name)
    n = fx["n"]
    prm = Params(lam=float(Fraction(fx["params"]["lambda"])),
                 beta_fast=float(Fraction(fx["params"]["beta_fast"])),
                 beta_slow=float(Fraction(fx["params"]["beta_slow"])), enable=True)
    x32 = np.zeros((2, n), F32)
    x32[0, :4] = [float(v) for v in _frac_list(fx["x"]["rank0"])]
    x32[1, :4] = [float(v) for v in _frac_list(fx["x"]["rank1"])]
    for x in (bf16_bits(x32), x32):
        f = np.zeros(n, F32)
        s = np.zeros(n, F32)
        for call in fx["calls"]:
            res = orc.allreduce(x, f, s, prm, want_diag=True, variant=variant)
            for key in ("c", "err", "f", "s", "out"):
                want = [Fraction(t) for t in call[key]] + [Fraction(0)] * (n - 4)
                have = {"c": res["c"], "err": res["err"], "f": f, "s": s,
                        "out": _values(res["out"])}[key]
                assert [Fraction(float(h)) for h in have] == want, (key, have[:4])
            assert res["codes1"][0, :2].tolist() == call["codes1_rank0"]
            assert res["codes1"][1, :2].tolist() == call["codes1_rank1"]
            assert not res["codes1"][:, 2:].any()
            assert res["scales1"].tolist() == call["scales1"]
            assert res["qcodes"][:2].tolist() == call["qcodes"]
            assert not res["qcodes"][2:].any()
            assert res["qscales"].tolist() == call["qscales"]


def pin_hand_example(orc):
    """Four calls of the hand-worked example (fixture
    ``hand_example_p2_g32.json``): every wire byte, output, correction, error
    and state value, for bf16 and binary32 inputs."""
    _check_hand_fixture(orc, "hand_example_p2_g32.json", 0)


def _dyadic(expr: str) -> Fraction:
    """``n*2^k``, ``n`` or ``p/q`` as an exact rational."""
    expr = expr.strip()
    if "*2^" in expr:
        coef, _, power = expr.partition("*2^")
        return Fraction(int(coef)) * Fraction(2) ** int(power)
    return Fraction(expr)


def _assert_nearest_binary32(exact: Fraction, rounded: Fraction, what: str):
    """``rounded`` is a binary32 value and no binary32 value lies nearer to
    ``exact``; on a tie the last significand bit of ``rounded`` is 0."""
    r = F32(float(rounded))
    assert Fraction(float(r)) == rounded, f"{what}: {rounded} is not a binary32 value"
    d = abs(exact - rounded)
    for nb in (np.nextafter(r, F32(-np.inf)), np.nextafter(r, F32(np.inf))):
        dn = abs(exact - Fraction(float(nb)))
        assert d <= dn, f"{what}: {float(nb)!r} is nearer to {exact} than {rounded}"
        if d == dn and d != 0:
            assert int(np.array(r).view(np.uint32)) & 1 == 0, f"{what}: tie not to even"


def _check_derivation(steps, vals, what):
    """Re-check each written step: its exact result from its operands, and
    its binary32 rounding. Adds every step's rounded result to ``vals``."""
    for st in steps:
        a = [vals[t] if t in vals else _dyadic(t) for t in st["args"]]
        exact = {"mul": lambda: a[0] * a[1], "add": lambda: a[0] + a[1],
                 "sub": lambda: a[0] - a[1], "fma": lambda: a[0] * a[1] + a[2]}[st["op"]]()
        assert exact == _dyadic(st["exact"]), (what, st)
        _assert_nearest_binary32(exact, _dyadic(st["rounded"]), f"{what}/{st['name']}")
        vals[st["name"]] = _dyadic(st["rounded"])


def pin_rounding_order(orc):
    """Hand-worked operation order (fixture ``rounding_order_p3_g32.json``):
    the correction c = RN(RN(lambda f) + RN((1-lambda) s)), each estimate
    RN(RN(beta z) + RN((1-beta) err)), and with sender feedback the owner's
    RN(RN(x + eps) + c), each product and sum rounded on its own. The probes
    are chosen so that fusing a product into the add, or reassociating the
    adds, changes the binary32 result; the fixture lists each such value. The
    pin re-checks every written step of the derivation (exact rational,
    nearest binary32), then requires the oracle's c, err, f, s, output and
    rank 0's new sender error at each probe, for bf16 and binary32 partials,
    under dyadic coefficients (5/8, 3/4, 7/8) and the binary32 values of
    0.25, 0.3, 0.95."""
    fx = _load("rounding_order_p3_g32.json")
    P, G = 3, 32
    m = P * G
    for case in fx["cases"]:
        prm = {k: _dyadic(v) for k, v in case["params"].items()}
        params = Params(lam=float(prm["lambda"]), beta_fast=float(prm["beta_fast"]),
                        beta_slow=float(prm["beta_slow"]))
        for k, v in prm.items():  # the coefficients themselves are binary32 values
            assert Fraction(float(F32(float(v)))) == v, (case["name"], k)
        variant = SENDER_EF if case["variant"] == "SENDER_EF" else 0
        x32 = np.zeros((P, m), F32)
        x32[0, 2] = 7.0
        x32[2, 0] = 12.0
        f0 = np.zeros(m, F32)
        s0 = np.zeros(m, F32)
        eps0 = np.zeros((P, m), F32)
        for p in case["probes"]:
            e = p["element"]
            assert 3 <= e < G
            x32[0, e] = 1.0
            x32[1, e] = 7.0 * 2.0 ** -10
            f0[e] = float(_dyadic(p["f"]))
            s0[e] = float(_dyadic(p["s"]))
            if "eps_rank0" in p:
                eps0[0, e] = float(_dyadic(p["eps_rank0"]))
        for p in case["probes"]:
            vals = {"lambda": prm["lambda"], "beta_fast": prm["beta_fast"],
                    "beta_slow": prm["beta_slow"], "f": _dyadic(p["f"]), "s": _dyadic(p["s"]),
                    "err": Fraction(-1017, 1024), "x": Fraction(1)}
            if "eps_rank0" in p:
                vals["eps"] = _dyadic(p["eps_rank0"])
            what = f"{case['name']}/{p['element']}"
            _check_derivation(p["steps"], vals, what)
            want = {k: _dyadic(v) for k, v in p["expect"].items()}
            assert want["err"] == vals["err"] and want["c"] == vals["c"]
            if "f" in want:
                assert want["f"] == vals["f_next"] and want["s"] == vals["s_next"]
            if "eps_rank0" in want:
                assert want["eps_rank0"] == vals["eps_next"]
            for alt in p["alternatives"]:
                avals = dict(vals)
                _check_derivation(alt["steps"], avals, f"{what}/{alt['mutant']}")
                assert _dyadic(alt["value"]) == avals[alt["steps"][-1]["name"]]
                key = "eps_rank0" if alt["of"] == "eps" else alt["of"]
                assert _dyadic(alt["value"]) != want[key], (what, alt["mutant"])
        for x in (x32, bf16_bits(x32)):
            f, s, eps = f0.copy(), s0.copy(), eps0.copy()
            res = orc.allreduce(x, f, s, params, want_diag=True, variant=variant,
                                eps=eps if variant else None)
            assert res["scales1"][:, 0].tolist() == [127, 117, 128]
            assert res["qscales"].tolist() == [128, 0, 0]
            q = _unpack_ref(res["qcodes"][:G // 2])
            assert q[0] == 6 and q[2] == 4
            for p in case["probes"]:
                e = p["element"]
                want = {k: _dyadic(v) for k, v in p["expect"].items()}
                assert _unpack_ref(res["codes1"][0][:G // 2])[e] == 1
                assert _unpack_ref(res["codes1"][1][:G // 2])[e] == 7
                assert q[e] == 1
                have = {"c": res["c"][e], "err": res["err"][e], "out": _values(res["out"])[e],
                        "f": f[e], "s": s[e], "eps_rank0": eps[0, e]}
                for key, w in want.items():
                    assert Fraction(float(have[key])) == w, (case["name"], e, key,
                                                             float(have[key]), float(w))


def _grid_partials(P, ngroups, G, seed):
    """Partials that rounding #1 reproduces exactly: each group is k*2^e_rg,
    |k| <= 7, with one |k| in 4..7 so that e_rg is the group's scale. Exponents
    stay within a span of 8 so binary32 sums are exact."""
    g = rng(seed, 31, P)
    e0 = int(g.integers(-40, 30))
    k = g.integers(-7, 8, (P, ngroups, G))
    lead = g.integers(0, G, (P, ngroups))
    sign = np.where(g.random((P, ngroups)) < 0.5, -1, 1)
    for r in range(P):
        for j in range(ngroups):
            k[r, j, lead[r, j]] = sign[r, j] * g.integers(4, 8)
    e = e0 + g.integers(0, 9, (P, ngroups))
    x = (k * np.exp2(e)[:, :, None].astype(np.float64)).astype(F32)
    return x.reshape(P, ngroups * G), k, e


def pin_exact_sums_on_grid(orc):
    """With partials already on their 4-bit grid, rounding #1 is exact, the sum
    is exact, and the result equals the exhaustive quantiser applied to the
    exact sum; err = exact sum - result. Covers P from 2 to 16, both dtypes,
    compensation off and a first call with it on (zero state); the group-size
    variants 16, 64 and 128 at P = 2 and 8."""
    cases = [(P, 32) for P in (2, 3, 4, 8, 16)] + [(P, G) for G in (16, 64, 128) for P in (2, 8)]
    for P, G in cases:
        ngroups = 2 * P
        m = ngroups * G
        x32, k, e = _grid_partials(P, ngroups, G, seed=P)
        exact = [sum(Fraction(float(x32[r, i])) for r in range(P)) for i in range(m)]
        want_Y, want_bytes = [], []
        for j in range(ngroups):
            b, q = bf_quantize([float(t) for t in exact[j * G:(j + 1) * G]])
            want_bytes.append(b)
            want_Y += [value_of(c, b) for c in q]
        for x in (x32, bf16_bits(x32)):
            for enable in (False, True):
                f = np.zeros(m, F32)
                s = np.zeros(m, F32)
                res = orc.allreduce(x, f, s, Params(enable=enable), G=G, want_diag=True)
                assert res["scales1"].tolist() == (e + 127).tolist()
                for r in range(P):
                    assert _unpack_ref(res["codes1"][r]) == k[r].reshape(-1).tolist()
                assert res["qscales"].tolist() == want_bytes
                out = [Fraction(float(t)) for t in _values(res["out"])]
                assert out == want_Y
                err = [Fraction(float(t)) for t in res["err"]]
                assert err == [a - b for a, b in zip(exact, want_Y)]


def pin_p2_enumeration(orc):
    """P = 2, every pair of codes (a, b) in [-7, 7]^2 at one position, with rank
    0 at scale 2^0 and rank 1 at 2^-1 (fixed by a 7 elsewhere in each group):
    the total a + b/2 is exact and the result is the exhaustive quantiser of the
    exact total (every tie of rounding #2 appears)."""
    G = 32
    pairs = [(a, b) for a in range(-7, 8) for b in range(-7, 8)]
    ngroups = 2 * len(pairs)      # pairs in segment 0, copies in segment 1
    m = ngroups * G
    x = np.zeros((2, m), F32)
    for j, (a, b) in enumerate(pairs * 2):
        x[0, j * G] = a
        x[0, j * G + 1] = 7
        x[1, j * G] = b * 0.5
        x[1, j * G + 1] = 3.5
    res = orc.allreduce(bf16_bits(x), params=Params(enable=False))
    out = _values(res["out"])
    for j, (a, b) in enumerate(pairs * 2):
        grp = [Fraction(a) + Fraction(b, 2), Fraction(21, 2)] + [Fraction(0)] * (G - 2)
        byte, q = bf_quantize([float(t) for t in grp])
        assert res["qscales"][j] == byte
        assert Fraction(float(out[j * G])) == value_of(q[0], byte), (a, b)
        assert Fraction(float(out[j * G + 1])) == value_of(q[1], byte)


def pin_rank_order(orc):
    """The owner adds in binary32, rank 0 first. Ranks 0, 1, 2 send 2^24, 1 and
    -2^24 (each exact after rounding #1): in that order binary32 gives
    (2^24 + 1) -> 2^24 (half to even), then 0; any other order, or a wider
    accumulator, gives 1."""
    G = 32
    P = 3
    m = P * G
    x = np.zeros((P, m), F32)
    x[0, 0] = 2.0 ** 24
    x[1, 0] = 1.0
    x[2, 0] = -(2.0 ** 24)
    for xx in (x, bf16_bits(x)):
        res = orc.allreduce(xx, params=Params(enable=False), want_diag=True)
        assert float(_values(res["out"])[0]) == 0.0
        assert float(res["err"][0]) == 0.0
        assert res["qscales"][0] == 0


def pin_owner_injection(orc):
    """Only the owner adds the correction, once, on its own contiguous segment.
    Zero partials and f = s = 3/4 everywhere: c = 3/4, so each rank's codes are
    6 at scale 2^-3 on its own segment and 0 elsewhere, every rank receives
    exactly 3/4, err = 0, then f = 3/8 and s = 21/32."""
    G = 32
    P = 4
    m = P * G * 2
    x = np.zeros((P, m), np.uint16)
    f = np.full(m, 0.75, F32)
    s = np.full(m, 0.75, F32)
    res = orc.allreduce(x, f, s, Params(), want_diag=True)
    seg = m // P
    for r in range(P):
        codes = _unpack_ref(res["codes1"][r])
        for i in range(m):
            assert codes[i] == (6 if i // seg == r else 0), (r, i)
        for j in range(m // G):
            assert res["scales1"][r, j] == (124 if (j * G) // seg == r else 0)
    assert (bf16_to_f32(res["out"]) == F32(0.75)).all()
    assert (res["err"] == 0).all()
    assert (f == F32(0.375)).all() and (s == F32(0.65625)).all()


def pin_degenerate(orc):
    """All-zero partials give scale byte 0, codes 0, output 0; opposite partials
    on two ranks cancel exactly (rounding is symmetric)."""
    G = 32
    P = 2
    m = P * G * 3
    zero = np.zeros((P, m), np.uint16)
    f = np.zeros(m, F32)
    s = np.zeros(m, F32)
    res = orc.allreduce(zero, f, s, Params(), want_diag=True)
    assert not res["codes1"].any() and not res["scales1"].any()
    assert not res["qcodes"].any() and not res["qscales"].any()
    assert not res["out"].any() and not f.any() and not s.any()
    x = gaussian(1, m, seed=3, call=0, dtype="fp32")[0]
    opp = np.stack([x, -x])
    res = orc.allreduce(opp, params=Params(enable=False), want_diag=True)
    c0 = _unpack_ref(res["codes1"][0])
    c1 = _unpack_ref(res["codes1"][1])
    assert c1 == [-c for c in c0]
    assert (res["out"] == 0).all() and (res["err"] == 0).all()


def pin_error_feedback_special_case(orc):
    """lambda = 1, beta_fast = 0 turns the compensator into textbook error
    feedback: the correction of call k is exactly the error captured in call
    k-1, so the running sum D_K = sum_{k<K} (c_k - err_k) telescopes to
    exactly -err_{K-1}."""
    P, G = 4, 32
    m = P * G * 4
    f = np.zeros(m, F32)
    s = np.zeros(m, F32)
    prm = Params(lam=1.0, beta_fast=0.0, beta_slow=0.875)
    cs, errs = [], []
    for k in range(12):
        res = orc.allreduce(gaussian(P, m, seed=5, call=k), f, s, prm, want_diag=True)
        cs.append(res["c"].astype(np.float64))
        errs.append(res["err"].astype(np.float64))
    assert not cs[0].any()
    for k in range(1, len(cs)):
        assert (cs[k] == errs[k - 1]).all()
    for K in range(1, len(cs) + 1):
        for i in range(0, m, 7):
            D = math.fsum([cs[k][i] - errs[k][i] for k in range(K)])
            assert D == -errs[K - 1][i]


def pin_bounded_partial_sum(orc):
    """Defaults (lambda = 1/2, beta_fast = 1/2, beta_slow = 7/8). The correction
    of call k is sum_j h_{k-1-j} err_j with sum_m h_m = 1, so
    D_K = -sum_j err_j * tail_{K-1-j}, tail_t = (beta_f^t + beta_s^t)/2, and
    |D_K| <= max|err| * (1/2/(1-1/2) + 1/2/(1-7/8)) = 5 max|err| for every K.
    Without compensation D_K = -sum err_k grows like sqrt(K)."""
    P, G, K = 4, 32, 96
    m = P * G * 8
    f = np.zeros(m, F32)
    s = np.zeros(m, F32)
    D_on = np.zeros(m)
    emax = np.zeros(m)
    D_off = np.zeros(m)
    for k in range(K):
        x = gaussian(P, m, seed=9, call=k)
        res = orc.allreduce(x, f, s, Params(), want_diag=True)
        D_on += res["c"].astype(np.float64) - res["err"].astype(np.float64)
        emax = np.maximum(emax, np.abs(res["err"].astype(np.float64)))
        assert (np.abs(D_on) <= 5.0 * emax * (1 + 1e-4) + 1e-30).all(), k
        off = orc.allreduce(x, params=Params(enable=False), want_diag=True)
        assert not off["c"].any()
        D_off -= off["err"].astype(np.float64)
    rms_on = math.sqrt(float(np.mean(D_on ** 2)))
    rms_off = math.sqrt(float(np.mean(D_off ** 2)))
    assert rms_on < 0.35 * rms_off, (rms_on, rms_off)


def pin_two_roundings_bound(orc):
    """Each element passes through at most two roundings whatever P:
    |Y - sum_r v_r| <= sum_r 2^(e_r - 1) + 2^(E - 1) + (P-1) * 2^-24 * sum_r |q_r 2^e_r|
    (the last term bounds the binary32 additions), with v_r the value rank r
    rounds (its partial, plus c at the owner)."""
    G = 32
    for P in (2, 8, 16):
        m = P * G * 2
        f = np.zeros(m, F32)
        s = np.zeros(m, F32)
        owner = np.arange(m) // (m // P)
        for k in range(4):
            x = gaussian(P, m, seed=P, call=k, dtype="fp32")
            x[:, ::97] *= 50
            res = orc.allreduce(x, f, s, Params(), want_diag=True)
            Y = res["out"].astype(np.float64)
            for i in range(0, m, 5):
                j = i // G
                total = Fraction(0)
                bound = Fraction(2) ** (int(res["qscales"][j]) - 128)
                mag = Fraction(0)
                for r in range(P):
                    v = x[r, i]
                    if owner[i] == r:
                        v = F32(v + res["c"][i])
                    total += Fraction(float(v))
                    b = int(res["scales1"][r, j])
                    q = _unpack_ref(res["codes1"][r][i // 2:i // 2 + 1])[i % 2]
                    bound += Fraction(2) ** (b - 128)
                    mag += abs(value_of(q, b))
                bound += (P - 1) * Fraction(1, 2 ** 24) * mag
                assert abs(Fraction(float(Y[i])) - total) <= bound, (P, k, i)


def pin_power_of_two_equivariance(orc):
    """Scaling every partial and the state by 2^t scales every output, error
    and state value by exactly 2^t and shifts every non-zero scale byte by t;
    the codes do not change."""
    P, G = 4, 32
    m = P * G * 4
    for dtype in ("bf16", "fp32"):
        for t in (-9, 13):
            f0, s0 = np.zeros(m, F32), np.zeros(m, F32)
            f1, s1 = np.zeros(m, F32), np.zeros(m, F32)
            for k in range(4):
                x = gaussian(P, m, seed=11, call=k, dtype="fp32")
                xs = (x * np.float32(2.0 ** t)).astype(F32)
                if dtype == "bf16":
                    x, xs = bf16_bits(x), bf16_bits(xs)
                a = orc.allreduce(x, f0, s0, Params(), want_diag=True)
                b = orc.allreduce(xs, f1, s1, Params(), want_diag=True)
                scale = F32(2.0 ** t)
                assert (_values(b["out"]) == _values(a["out"]) * scale).all()
                assert (b["err"] == a["err"] * scale).all()
                assert (f1 == f0 * scale).all() and (s1 == s0 * scale).all()
                assert (a["codes1"] == b["codes1"]).all() and (a["qcodes"] == b["qcodes"]).all()
                nz = a["scales1"] != 0
                assert (b["scales1"][nz].astype(int) == a["scales1"][nz].astype(int) + t).all()
                nzq = a["qscales"] != 0
                assert (b["qscales"][nzq].astype(int) == a["qscales"][nzq].astype(int) + t).all()


# ---------------------------------------------------------------------------
# variants: the correction folded into the owner's sum; sender-side feedback
# ---------------------------------------------------------------------------
def pin_owner_sum_hand_example(orc):
    """Three calls of the hand-worked owner-sum example (fixture
    ``hand_example_owner_sum_p2_g32.json``): the senders' wire never changes,
    the correction enters the owner's sum exactly."""
    _check_hand_fixture(orc, "hand_example_owner_sum_p2_g32.json", OWNER_SUM)


def pin_owner_sum_injection(orc):
    """Owner-sum variant: zero partials and f = s = 3/4. No sender adds
    anything (all stage-1 codes and scale bytes are 0); the owner's sum is
    exactly 3/4 everywhere, so every rank receives 3/4 with err = 0."""
    G, P = 32, 4
    m = P * G * 2
    f = np.full(m, 0.75, F32)
    s = np.full(m, 0.75, F32)
    res = orc.allreduce(np.zeros((P, m), np.uint16), f, s, Params(), want_diag=True,
                        variant=OWNER_SUM)
    assert not res["codes1"].any() and not res["scales1"].any()
    assert (bf16_to_f32(res["out"]) == F32(0.75)).all()
    assert (res["qscales"] == 124).all() and (res["err"] == 0).all()
    assert (f == F32(0.375)).all() and (s == F32(0.65625)).all()


def pin_owner_sum_order(orc):
    """Owner-sum variant: the correction is added after the P restored values.
    Ranks send 2^24 and -2^24 (exact) and c = 1: (2^24 - 2^24) + 1 = 1,
    whereas starting the sum from c would give (1 + 2^24) -> 2^24, then 0."""
    G, P = 32, 2
    m = P * G
    x = np.zeros((P, m), F32)
    x[0, 0] = 2.0 ** 24
    x[1, 0] = -(2.0 ** 24)
    f = np.ones(m, F32)
    s = np.ones(m, F32)
    res = orc.allreduce(x, f, s, Params(), want_diag=True, variant=OWNER_SUM)
    assert float(res["out"][0]) == 1.0 and float(res["err"][0]) == 0.0
    assert (res["out"][1:G] == 1.0).all()


def pin_owner_sum_error_feedback(orc):
    """Owner-sum variant with lambda = 1, beta_fast = 0 (textbook error
    feedback): c_k = err_{k-1} exactly and D_K = -err_{K-1} exactly."""
    P, G = 4, 32
    m = P * G * 4
    f = np.zeros(m, F32)
    s = np.zeros(m, F32)
    prm = Params(lam=1.0, beta_fast=0.0, beta_slow=0.875)
    cs, errs = [], []
    for k in range(10):
        res = orc.allreduce(gaussian(P, m, seed=15, call=k), f, s, prm, want_diag=True,
                            variant=OWNER_SUM)
        cs.append(res["c"].astype(np.float64))
        errs.append(res["err"].astype(np.float64))
    for k in range(1, len(cs)):
        assert (cs[k] == errs[k - 1]).all()
    for i in range(0, m, 11):
        assert math.fsum([cs[k][i] - errs[k][i] for k in range(len(cs))]) == -errs[-1][i]


def pin_sender_ef_on_grid(orc):
    """Sender feedback on partials already on their 4-bit grid: rounding #1
    is exact, so every rank's stored error stays exactly 0 and the results
    equal those without the feedback."""
    G = 32
    for P in (2, 5, 8):
        ngroups = 2 * P
        m = ngroups * G
        x32, _, _ = _grid_partials(P, ngroups, G, seed=40 + P)
        eps = np.zeros((P, m), F32)
        a = orc.allreduce(x32, params=Params(enable=False), want_diag=True, variant=SENDER_EF,
                          eps=eps)
        b = orc.allreduce(x32, params=Params(enable=False), want_diag=True)
        assert not eps.any()
        assert (a["out"] == b["out"]).all() and (a["codes1"] == b["codes1"]).all()


def pin_sender_ef_per_rank(orc):
    """Each rank keeps its own error: only the rank whose partial is off its
    grid gets a non-zero error, equal to v - q*2^e exactly, at most half a
    step; the next call adds it to that rank's partial only."""
    G, P = 32, 4
    m = P * G
    x = np.zeros((P, m), F32)
    x[:, 0] = 7.0          # every group's maximum: scale 2^0 on every rank
    x[2, 1] = 0.3          # rank 2, element 1: rounds to 0, error 0.3
    x[1, 2] = 2.0          # on the grid
    eps = np.zeros((P, m), F32)
    orc.allreduce(x, params=Params(enable=False), variant=SENDER_EF, eps=eps)
    assert eps[2, 1] == F32(0.3)
    eps_rest = eps.copy()
    eps_rest[2, 1] = 0
    assert not eps_rest.any()
    # next call: rank 2 forms 0.3 + 0.3 = 0.6 (binary32), rounds to 1, error -0.4
    res = orc.allreduce(x, params=Params(enable=False), variant=SENDER_EF, eps=eps)
    assert eps[2, 1] == F32(F32(0.3) + F32(0.3)) - F32(1.0)
    assert _unpack_ref(res["codes1"][2][:1])[1] == 1
    eps_rest = eps.copy()
    eps_rest[2, 1] = 0
    assert not eps_rest.any()


def pin_full_compensation_bounded(orc):
    """With both roundings fed back (sender feedback, and the owner's
    correction either at the sender or in the sum) the total injected error
    telescopes: T_K = sum_k (Y_k - sum_r x_rk) = D_K - sum_r eps_r,K-1 + R_K,
    |D_K| <= 5 max|err| (closed form), R_K the binary32 rounding of the sums
    (at most ulp-sized per term). So T_K stays bounded however many calls, while
    with the owner's correction alone it grows like sqrt(K) (stage-1 errors)."""
    P, G, K = 4, 32, 96
    m = P * G * 8
    rms = {}
    for variant in (SENDER_EF, SENDER_EF | OWNER_SUM, 0):
        f = np.zeros(m, F32)
        s = np.zeros(m, F32)
        eps = np.zeros((P, m), F32)
        T = np.zeros(m)
        emax = np.zeros(m)
        epsmax = np.zeros(m)
        xmax = np.zeros(m)
        for k in range(K):
            x = gaussian(P, m, seed=13, call=k, dtype="fp32")
            res = orc.allreduce(x, f, s, Params(), want_diag=True, variant=variant, eps=eps)
            T += res["out"].astype(np.float64) - x.astype(np.float64).sum(axis=0)
            emax = np.maximum(emax, np.abs(res["err"]))
            xmax = np.maximum(xmax, np.abs(x).sum(axis=0) + 8)
            if variant & SENDER_EF:
                epsmax = np.maximum(epsmax, np.abs(eps).max(axis=0))
                bound = 5 * emax + P * epsmax + (k + 1) * 4 * P * 2.0 ** -23 * xmax
                assert (np.abs(T) <= bound).all(), (variant, k)
        rms[variant] = math.sqrt(float(np.mean(T ** 2)))
    assert rms[SENDER_EF] < 0.3 * rms[0], rms
    assert rms[SENDER_EF | OWNER_SUM] < 0.3 * rms[0], rms


# ---------------------------------------------------------------------------
# binary16-scale variant (scale = the smallest binary16 s with 7*s >= max|v|)
# ---------------------------------------------------------------------------
def _f16_groups(count, G, seed):
    """Random groups plus the cases the binary16 rule turns on: 7*s exactly
    at the maximum, one ulp past it, the subnormal binary16 range, below the
    smallest binary16 step, past the largest scale (saturation), zero."""
    groups = _random_groups(count, G, seed)
    g = rng(seed, 16)
    for h in (0x3C00, 0x0001, 0x0200, 0x03FF, 0x0400, 0x2E66, 0x7BFF, 0x5A5A):
        sv = float(half_fraction(h))
        v = g.uniform(-7, 7, G) * sv
        v[0] = 7 * sv                                   # exactly 7*s: s itself
        groups.append(v.astype(F32))
        w = v.astype(F32)
        w[1] = np.nextafter(F32(7 * sv), F32(np.inf))   # just past: the next binary16
        groups.append(w)
        t = (g.integers(-7, 8, G) + 0.5) * sv           # exact ties k + 1/2
        t[0] = 7 * sv
        groups.append(t.astype(F32))
    groups.append((g.standard_normal(G) * 1e6).astype(F32))      # saturates at 65504
    groups.append((g.standard_normal(G) * 2.0 ** -30).astype(F32))  # below 2^-24
    groups.append(np.zeros(G, F32))
    return groups


def pin_f16_quantizer_bruteforce(orc):
    """Binary16 scale pattern and every code equal an exhaustive search over
    all binary16 scales (decoded by numpy) and all codes, with exact
    distances; ties go to the even code."""
    for G in (32, 16, 2):
        for v in _f16_groups(36 if G == 32 else 12, G, seed=200 + G):
            h, q = orc.quantize_group_f16(v)
            bh, bq = bf_quantize_f16(v.tolist())
            assert h == bh, (v, h, bh)
            assert q.tolist() == bq, (v, q.tolist(), bq)


def pin_f16_values(orc):
    """Restored values are q*s exactly (numpy's binary16 decoding); the bf16
    rounding of outputs agrees with the bit-pattern rule add-0x7FFF-plus-odd;
    a restored q*s is within s/2 of v unless the scale saturated, and s is
    within one binary16 step of max|v|/7."""
    for h in list(range(1, 0x7C00, 97)) + [0x7BFF, 1, 0x3FF, 0x400]:
        sv = half_fraction(h)
        assert Fraction(orc.half_value(h)) == sv
        for q in range(-7, 8):
            y = orc.dequant_f16(q, h)
            assert Fraction(y) == q * sv
            assert orc.round_bf16(y) == bf16_round_bits(y), (q, h)
    g = rng(5, 16)
    for x in np.concatenate([g.standard_normal(4000) * 2.0 ** g.integers(-30, 20, 4000),
                             (g.integers(0, 2 ** 16, 500) * 2.0 + 1) * 2.0 ** -16]).astype(F32):
        assert orc.round_bf16(float(x)) == bf16_round_bits(float(x)), x
    for v in _f16_groups(12, 32, seed=7):
        h, q = orc.quantize_group_f16(v)
        A = max(abs(Fraction(float(t))) for t in v)
        if A == 0:
            continue
        sv = half_fraction(h)
        if A <= 7 * Fraction(65504):
            assert 7 * sv >= A and (h == 1 or 7 * half_fraction(h - 1) < A)
            for t, k in zip(v, q.tolist()):
                assert abs(Fraction(float(t)) - k * sv) <= sv / 2


def _f16_grid_partials(P, ngroups, G, seed):
    """Partials k*s with s a binary16 and one |k| = 7 per group, so that
    rounding #1 reproduces them exactly with scale s. The scales stay within a
    narrow range so that binary32 sums are exact."""
    g = rng(seed, 161, P)
    k = g.integers(-7, 8, (P, ngroups, G))
    lead = g.integers(0, G, (P, ngroups))
    h = g.integers(0x3800, 0x3C00, (P, ngroups)).astype(np.uint16)   # s in [0.5, 1)
    for r in range(P):
        for j in range(ngroups):
            k[r, j, lead[r, j]] = 7 if g.random() < 0.5 else -7
    sv = h.view(np.float16).astype(np.float64)
    x = (k * sv[:, :, None]).astype(F32)
    return x.reshape(P, ngroups * G), k, h


def pin_f16_exact_sums_on_grid(orc):
    """Binary16 scales with partials on their grid: rounding #1 is exact, the
    binary32 sum is exact, the total is the exhaustive quantiser's result on
    the exact sum; a binary32 output is q*s exactly, a bf16 output is that
    rounded to the nearest bf16 (ties to even), and the captured error is the
    exact sum minus what the ranks receive."""
    for P, G in [(2, 32), (5, 32), (8, 16), (3, 128)]:
        ngroups = 2 * P
        m = ngroups * G
        x32, k, h = _f16_grid_partials(P, ngroups, G, seed=P * G)
        exact = [sum(Fraction(float(x32[r, i])) for r in range(P)) for i in range(m)]
        want_h, want_Y = [], []
        for j in range(ngroups):
            bh, bq = bf_quantize_f16([float(t) for t in exact[j * G:(j + 1) * G]])
            want_h.append(bh)
            want_Y += [c * half_fraction(bh) for c in bq]
        for x, bf in ((x32, False), (bf16_bits(x32), True)):
            if bf and not (bf16_to_f32(x) == x32).all():
                continue   # k*s is not always a bf16: that input would round first
            for enable in (False, True):
                f = np.zeros(m, F32)
                s = np.zeros(m, F32)
                res = orc.allreduce(x, f, s, Params(enable=enable), G=G, want_diag=True,
                                    variant=FP16_SCALE)
                assert res["scales1"].tolist() == h.tolist()
                for r in range(P):
                    assert _unpack_ref(res["codes1"][r]) == k[r].reshape(-1).tolist()
                assert res["qscales"].tolist() == want_h
                Y = [Fraction(bf16_round_bits(float(y))) if bf else y for y in want_Y]
                out = [Fraction(float(t)) for t in _values(res["out"])]
                assert out == Y
                err = [Fraction(float(t)) for t in res["err"]]
                assert err == [a - b for a, b in zip(exact, Y)]
        # bf16 inputs that are on a bf16 grid: k*s with s = 2^j * (1 + i/8)
        hb = (0x3800 + (np.arange(ngroups * P) % 8) * 128).astype(np.uint16).reshape(P, ngroups)
        xb = (k * hb.view(np.float16).astype(np.float64)[:, :, None]).astype(F32).reshape(P, m)
        assert (bf16_to_f32(bf16_bits(xb)) == xb).all()
        res = orc.allreduce(bf16_bits(xb), params=Params(enable=False), G=G, want_diag=True,
                            variant=FP16_SCALE)
        assert res["scales1"].tolist() == hb.tolist()
        exact = [sum(Fraction(float(xb[r, i])) for r in range(P)) for i in range(m)]
        for j in range(ngroups):
            bh, bq = bf_quantize_f16([float(t) for t in exact[j * G:(j + 1) * G]])
            assert res["qscales"][j] == bh
            for t in range(G):
                y = Fraction(bf16_round_bits(float(bq[t] * half_fraction(bh))))
                i = j * G + t
                assert Fraction(float(_values(res["out"])[i])) == y
                assert Fraction(float(res["err"][i])) == exact[i] - y


def pin_f16_feedback(orc):
    """The compensator and both feedback variants run unchanged over binary16
    scales: with lambda = 1, beta_fast = 0 the correction of call k is
    exactly the error of call k-1; sender feedback on grid partials keeps
    every stored error at 0; the closed-form bound |D_K| <= 5 max|err| holds."""
    P, G = 4, 32
    m = P * G * 4
    f = np.zeros(m, F32)
    s = np.zeros(m, F32)
    prev = None
    for k in range(8):
        res = orc.allreduce(gaussian(P, m, seed=6, call=k), f, s, Params(lam=1.0, beta_fast=0.0),
                            want_diag=True, variant=FP16_SCALE)
        if prev is not None:
            assert (res["c"] == prev).all()
        prev = res["err"].copy()
    x32, _, _ = _f16_grid_partials(P, 2 * P, G, seed=77)
    eps = np.zeros((P, x32.shape[1]), F32)
    orc.allreduce(x32, params=Params(enable=False), variant=FP16_SCALE | SENDER_EF, eps=eps)
    assert not eps.any()
    f = np.zeros(m, F32)
    s = np.zeros(m, F32)
    D = np.zeros(m)
    emax = np.zeros(m)
    for k in range(48):
        res = orc.allreduce(gaussian(P, m, seed=8, call=k), f, s, Params(), want_diag=True,
                            variant=FP16_SCALE)
        D += res["c"].astype(np.float64) - res["err"].astype(np.float64)
        emax = np.maximum(emax, np.abs(res["err"].astype(np.float64)))
        assert (np.abs(D) <= 5.0 * emax * (1 + 1e-4) + 1e-30).all(), k


def _many_random_groups(ngroups, G, seed):
    """Groups of random magnitudes (2^-140 .. 2^100 per group, with
    subnormals, ties on a power-of-two grid and bf16 values mixed in)."""
    g = rng(seed, 77, ngroups)
    x = g.standard_normal((ngroups, G)) * np.exp2(g.integers(-140, 100, (ngroups, 1)).astype(np.float64))
    tie_rows = g.random(ngroups) < 0.2     # halves on a power-of-two grid
    e = g.integers(-120, 100, (ngroups, 1)).astype(np.float64)
    ties = (g.integers(-7, 7, (ngroups, G)) + 0.5) * np.exp2(e)
    ties[:, 0] = 7 * np.exp2(e[:, 0])
    x = np.where(tie_rows[:, None], ties, x)
    x = x.astype(np.float32)
    bf_rows = g.random(ngroups) < 0.2
    x[bf_rows] = bf16_to_f32(bf16_bits(x[bf_rows]))
    return x


def _quantise_rows_with_oracle(orc, x, G, variant):
    """Stage-1 codes and scales of rank 0 for the rows of x (compensation off,
    so rank 0 rounds exactly its own values), through one oracle call."""
    ngroups = x.shape[0]
    P = 2
    xs = np.stack([x.reshape(-1), np.zeros(ngroups * G, np.float32)])
    owner = np.zeros(ngroups, np.int32)
    res = orc.allreduce(xs, params=Params(enable=False), G=G, owner=owner, variant=variant)
    codes = np.array(_unpack_ref(res["codes1"][0])).reshape(ngroups, G)
    return res["scales1"][0].astype(np.int64), codes


def pin_quantizer_many_groups(orc):
    """About a million random groups through the oracle's rounding #1 against
    the vectorised exhaustive search: every scale byte and every code; and a
    quarter of that many through the binary16-scale rounding."""
    x = _many_random_groups(1 << 20, 32, seed=1)
    b, q = _quantise_rows_with_oracle(orc, x, 32, 0)
    bb, bq = bf_quantize_many(x)
    bad = np.flatnonzero((b != bb) | (q != bq).any(axis=1))
    assert bad.size == 0, (bad[:5], x[bad[:1]], b[bad[:1]], bb[bad[:1]])
    x = _many_random_groups(1 << 18, 32, seed=2)
    x = np.clip(x, -1e6, 1e6).astype(np.float32)  # include saturated groups, stay finite
    h, q = _quantise_rows_with_oracle(orc, x, 32, FP16_SCALE)
    bh, bq = bf_quantize_f16_many(x)
    bad = np.flatnonzero((h != bh) | (q != bq).any(axis=1))
    assert bad.size == 0, (bad[:5], x[bad[:1]], h[bad[:1]], bh[bad[:1]])


ALL_PINS = [
    pin_scale_boundaries,
    pin_quantizer_bruteforce,
    pin_roundtrip_bound,
    pin_pack_layout,
    pin_hand_example,
    pin_rounding_order,
    pin_exact_sums_on_grid,
    pin_p2_enumeration,
    pin_rank_order,
    pin_owner_injection,
    pin_degenerate,
    pin_error_feedback_special_case,
    pin_bounded_partial_sum,
    pin_two_roundings_bound,
    pin_power_of_two_equivariance,
    pin_owner_sum_hand_example,
    pin_owner_sum_injection,
    pin_owner_sum_order,
    pin_owner_sum_error_feedback,
    pin_sender_ef_on_grid,
    pin_sender_ef_per_rank,
    pin_full_compensation_bounded,
    pin_f16_quantizer_bruteforce,
    pin_f16_values,
    pin_f16_exact_sums_on_grid,
    pin_f16_feedback,
    pin_quantizer_many_groups,
]
