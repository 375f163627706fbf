"""Binary16-scale variant (ECHO_VARIANT_FP16_SCALE), CUDA path against the
oracle bit for bit.

Each group's scale is the smallest positive finite binary16 s with
7*s >= max|v|, codes are the nearest integers to v/s in [-7, 7] (ties to
even), bf16 outputs are q*s rounded to the nearest bf16 and the owner's error
is taken against that received value. The pages leave the scale format open
[rit.work "Echo 4-bit GPU communication", section "How Echo returns the error
to later calls": 4-bit integer segments]; this is the finer, costlier
alternative to power-of-two scale bytes.

Compared after every call: both wires (binary16 scale patterns included),
every rank's output, both phases' f and s, every rank's sender error.
"""
import numpy as np
import pytest

from bit_error_compensated_rank_b200 import workloads as wl
from bit_error_compensated_rank_b200.workloads import bf16_bits, gaussian, outlier_gaussian, rng
from gpu_harness import FullCompare, SampledCompare, assert_same_bits
from oracle.oracle import FP16_SCALE, OWNER_SUM, SENDER_EF, Params

pytestmark = pytest.mark.gpu


def _n(P, G, k):
    n = P * G * k
    return n if n % 32 == 0 else 2 * n


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("P,k", [(2, 37), (8, 41), (16, 9), (5, 3)])
@pytest.mark.parametrize("G", [32, 16, 64, 128])
def test_fp16_scale_sequences(oracle, G, P, k, dtype):
    n = _n(P, G, k)
    fc = FullCompare(oracle, P, n, dtype, group=G, variant=FP16_SCALE)
    try:
        for c, ph in enumerate([0, 0, 1, 0, 1]):
            fc.call(outlier_gaussian(P, n, seed=80 + P, call=c, dtype=dtype), phase=ph)
    finally:
        fc.close()


@pytest.mark.parametrize("variant", [OWNER_SUM, SENDER_EF, OWNER_SUM | SENDER_EF],
                         ids=["owner_sum", "sender_ef", "both"])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_fp16_scale_with_feedback_variants(oracle, variant, dtype):
    P, n = 4, 4 * 32 * 29
    fc = FullCompare(oracle, P, n, dtype, variant=variant | FP16_SCALE)
    try:
        for c in range(5):
            fc.call(outlier_gaussian(P, n, seed=81, call=c, dtype=dtype), phase=c & 1)
    finally:
        fc.close()


def _edge(kind, P, n, G):
    g = rng(23, len(kind), G)
    if kind == "saturating":     # beyond 7 * 65504: codes saturate at +-7
        x = g.standard_normal((P, n)) * 2.0 ** 20
    elif kind == "tiny":         # below the smallest binary16 step
        x = g.standard_normal((P, n)) * 2.0 ** -28
    elif kind == "subnormal":    # binary32 subnormals: every group rounds to zero
        x = g.integers(-2 ** 20, 2 ** 20, (P, n)) * 2.0 ** -149
    elif kind == "ties":         # exact midpoints (k + 1/2) * s of binary16 scales
        h = g.integers(0x2000, 0x5000, (P, n // G)).astype(np.uint16)
        s = np.repeat(h.view(np.float16).astype(np.float64), G, axis=1)
        k = g.integers(-7, 7, (P, n)) + 0.5
        k[:, ::G] = 7
        x = k * s
    elif kind == "near_ties":    # up to 6 binary32 ulps either side of the midpoints (k + 1/2) * s
        h = g.integers(0x2000, 0x5000, (P, n // G)).astype(np.uint16)
        s = np.repeat(h.view(np.float16).astype(np.float64), G, axis=1)
        k = g.integers(-7, 7, (P, n)) + 0.5
        k[:, ::G] = 7
        x = (k * s).astype(np.float32)
        off = g.integers(-6, 7, (P, n)).astype(np.int32)
        off[:, ::G] = 0  # keeps each group's maximum at exactly 7*s
        x = (x.view(np.int32) + off).view(np.float32)
    elif kind == "boundary":     # max|v| exactly 7*s and one ulp past it
        h = g.integers(0x0400, 0x7000, (P, n // G)).astype(np.uint16)
        s = np.repeat(h.view(np.float16).astype(np.float64), G, axis=1)
        x = g.uniform(-6.9, 6.9, (P, n)) * s
        x[:, ::G] = 7 * s[:, ::G]
        x = x.astype(np.float32)
        x[:, 1::2 * G] = np.nextafter(x[:, ::2 * G], np.float32(np.inf))
    elif kind == "zeros":
        x = np.zeros((P, n))
    else:
        raise ValueError(kind)
    return np.asarray(x, np.float64).astype(np.float32)


@pytest.mark.parametrize("kind", ["saturating", "tiny", "subnormal", "ties", "near_ties", "boundary", "zeros"])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_fp16_scale_edge_values(oracle, kind, dtype):
    P, G = 4, 32
    n = P * G * 24
    params = Params(enable=kind not in ("saturating",))  # saturated errors would grow the state
    fc = FullCompare(oracle, P, n, dtype, params=params, variant=FP16_SCALE)
    try:
        for c in range(3):
            x = _edge(kind, P, n, G) * np.float32(1 + c / 16)
            fc.call(bf16_bits(x) if dtype == "bf16" else x)
    finally:
        fc.close()


def test_fp16_scale_switching_formats(oracle):
    """Scale formats can change between calls; the state carries over."""
    P, n = 4, 4 * 32 * 50
    fc = FullCompare(oracle, P, n, "bf16")
    try:
        for c, variant in enumerate([0, FP16_SCALE, FP16_SCALE, 0, FP16_SCALE | OWNER_SUM, 0]):
            if variant != fc.variant:
                fc.h.set_variant(variant)
                fc.variant = variant
            fc.call(gaussian(P, n, seed=14, call=c))
    finally:
        fc.close()


@pytest.mark.parametrize("G", [32, 128])
def test_fp16_scale_at_one_gib(oracle, G):
    """The benchmark's size (P = 8, 1 GiB bf16 per rank), sampled blocks."""
    import torch
    P, n = 8, 1 << 29
    sc = SampledCompare(oracle, P, n, "bf16", group=G, variant=FP16_SCALE)
    try:
        bufs = [torch.empty(n, device="cuda", dtype=torch.bfloat16) for _ in range(P)]
        for c in range(3):
            for r in range(P):
                wl.torch_outlier_gaussian_(bufs[r], seed=15, call=c, rank=r)
            sc.call(bufs, phase=c & 1)
    finally:
        sc.close()
        del bufs
        torch.cuda.empty_cache()


def test_fp16_scale_host_end_to_end(oracle):
    import torch
    from bit_error_compensated_rank_b200 import echo
    P, n = 4, 4 * 32 * 80000
    h = echo.Echo(P, n)
    h.set_variant(echo.ECHO_VARIANT_FP16_SCALE)
    try:
        f = np.zeros(n, np.float32)
        s = np.zeros(n, np.float32)
        for c in range(2):
            x = gaussian(P, n, seed=16, call=c)
            host_in = [torch.from_numpy(x[r].view(np.int16)).view(torch.bfloat16).pin_memory()
                       for r in range(P)]
            host_out = torch.empty(n, dtype=torch.bfloat16).pin_memory()
            h.allreduce_host(host_in, host_out)
            ref = oracle.allreduce(x, f, s, Params(), variant=FP16_SCALE)
            assert_same_bits(host_out.view(torch.int16).numpy().view(np.uint16), ref["out"], "host result")
            gf, gs = h.get_state(0)
            assert_same_bits(gf, f, "fast estimate")
            assert_same_bits(gs, s, "slow estimate")
    finally:
        h.close()
