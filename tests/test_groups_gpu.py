"""Group-size variants (16, 64 and 128 elements per power-of-two scale), CUDA
path against the oracle bit for bit.

The pages fix 32 elements per scale for the 4-bit segments [rit.work "Echo
4-bit GPU communication", section "How Echo returns the error to later
calls"]; smaller groups follow outliers more closely, larger ones spend fewer
scale bytes. Everything else (scale rule, rounding, owner layout, feedback)
is unchanged, so the oracle runs with the same G and both sides must agree
on every wire byte, output, state value and sender error.
"""
import numpy as np
import pytest

from bit_error_compensated_rank_b200 import workloads as wl
from bit_error_compensated_rank_b200.workloads import bf16_bits, gaussian, outlier_gaussian, rng
from gpu_harness import FullCompare, SampledCompare, assert_same_bits
from oracle.oracle import OWNER_SUM, SENDER_EF, Params

pytestmark = pytest.mark.gpu

GROUPS = [16, 64, 128]


def _n(P, G, k):
    """P*G*k elements, rounded up so that n is a multiple of 32 as well."""
    n = P * G * k
    return n if n % 32 == 0 else 2 * n


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("P,k", [(2, 37), (8, 41), (16, 9), (5, 3), (3, 1)])
@pytest.mark.parametrize("G", GROUPS)
def test_group_sequences(oracle, G, P, k, dtype):
    n = _n(P, G, k)
    fc = FullCompare(oracle, P, n, dtype, group=G)
    try:
        for c, ph in enumerate([0, 0, 1, 0, 1]):
            fc.call(outlier_gaussian(P, n, seed=60 + P, call=c, dtype=dtype), phase=ph)
    finally:
        fc.close()


@pytest.mark.parametrize("G", GROUPS)
@pytest.mark.parametrize("variant", [OWNER_SUM, SENDER_EF, OWNER_SUM | SENDER_EF],
                         ids=["owner_sum", "sender_ef", "both"])
def test_group_variants(oracle, G, variant):
    P = 4
    n = _n(P, G, 23)
    fc = FullCompare(oracle, P, n, "bf16", group=G, variant=variant)
    try:
        for c in range(4):
            fc.call(outlier_gaussian(P, n, seed=70, call=c), phase=c & 1)
    finally:
        fc.close()


@pytest.mark.parametrize("G", GROUPS)
def test_group_out_of_place_and_params(oracle, G):
    P = 8
    n = _n(P, G, 19)
    for params in (Params(), Params(lam=0.25, beta_fast=0.75, beta_slow=0.9375), Params(enable=False)):
        fc = FullCompare(oracle, P, n, "fp32", params=params, group=G)
        try:
            for c in range(3):
                fc.call(gaussian(P, n, seed=5, call=c, dtype="fp32"), out_of_place=True)
        finally:
            fc.close()


@pytest.mark.parametrize("G", GROUPS)
@pytest.mark.parametrize("kind", ["ties", "one_outlier", "subnormal", "huge"])
def test_group_edge_values(oracle, G, kind):
    P = 4
    n = _n(P, G, 12)
    g = rng(19, G, len(kind))
    if kind == "ties":
        x = g.integers(-7, 7, (P, n)) + 0.5
        x[:, ::G] = 7
        x = x * 2.0 ** g.integers(-20, 20, (P, 1))
    elif kind == "one_outlier":
        x = g.standard_normal((P, n))
        x[:, 5::G] *= 1000
    elif kind == "subnormal":
        x = g.integers(-2 ** 20, 2 ** 20, (P, n)) * 2.0 ** -149
    else:
        x = g.standard_normal((P, n)) * 2.0 ** 100
    x = x.astype(np.float32)
    fc = FullCompare(oracle, P, n, "bf16", group=G)
    try:
        for c in range(3):
            fc.call(bf16_bits(x * np.float32(1 + c / 8)))
    finally:
        fc.close()


@pytest.mark.parametrize("G", [16, 128])
def test_group_at_one_gib(oracle, G):
    """The benchmark's size (P = 8, 1 GiB bf16 per rank), sampled blocks."""
    import torch
    P, n = 8, 1 << 29
    sc = SampledCompare(oracle, P, n, "bf16", group=G, variant=OWNER_SUM | SENDER_EF if G == 16 else 0)
    try:
        bufs = [torch.empty(n, device="cuda", dtype=torch.bfloat16) for _ in range(P)]
        for c in range(3):
            for r in range(P):
                wl.torch_outlier_gaussian_(bufs[r], seed=11, call=c, rank=r)
            sc.call(bufs, phase=c & 1)
    finally:
        sc.close()
        del bufs
        torch.cuda.empty_cache()


@pytest.mark.parametrize("G", [16, 128])
def test_group_host_end_to_end(oracle, G):
    """Host buffers in, host result out, over several pipelined pieces."""
    import torch
    from bit_error_compensated_rank_b200 import echo
    P, n = 4, 4 * 128 * 20000  # 10.24 M elements per rank
    h = echo.Echo(P, n, echo.ECHO_BF16, G)
    try:
        f = np.zeros(n, np.float32)
        s = np.zeros(n, np.float32)
        for c in range(2):
            x = gaussian(P, n, seed=12, call=c)
            host_in = [torch.from_numpy(x[r].view(np.int16)).view(torch.bfloat16).pin_memory()
                       for r in range(P)]
            host_out = torch.empty(n, dtype=torch.bfloat16).pin_memory()
            h.allreduce_host(host_in, host_out)
            ref = oracle.allreduce(x, f, s, Params(), G=G)
            assert_same_bits(host_out.view(torch.int16).numpy().view(np.uint16), ref["out"], "host result")
            gf, gs = h.get_state(0)
            assert_same_bits(gf, f, "fast estimate")
            assert_same_bits(gs, s, "slow estimate")
    finally:
        h.close()


def test_group_wire_size():
    """The stage-1 and requantised wires carry n/G scale bytes."""
    from bit_error_compensated_rank_b200 import echo
    P = 4
    for G in (16, 32, 64, 128):
        n = P * 128 * 3
        h = echo.Echo(P, n, echo.ECHO_BF16, G)
        try:
            import torch
            bufs = [torch.randn(n, device="cuda").to(torch.bfloat16) for _ in range(P)]
            h.allreduce(bufs)
            torch.cuda.synchronize()
            codes, scales = h.get_wire(2)
            assert codes.size == n // 2 and scales.size == n // G
            assert (scales > 100).all()  # N(0, 1) data: scale exponents near 0
        finally:
            h.close()
