"""The one-kernel path (kf_fused_allreduce, chosen by echo_set_fused_limit)
against the CPU oracle bit for bit, and against the three pipelined kernels on
the same inputs.

Compared after every call, as in the other parity tests: every rank's stage-1
codes and scales, the requantised wire, every rank's output, both phases' f
and s, and every rank's sender errors. The shapes leave ragged warps (n/8 not
a multiple of 32 chunks) and groups that straddle no warp."""
import numpy as np
import pytest

from bit_error_compensated_rank_b200.workloads import bf16_bits, gaussian, outlier_gaussian
from gpu_harness import FullCompare, assert_same_bits
from oracle.oracle import FP16_SCALE, OWNER_SUM, SENDER_EF, Params
from test_fp16_scale_gpu import _edge as _fp16_edge
from test_parity_gpu import _edge_inputs

pytestmark = pytest.mark.gpu

SHAPES = [(2, 2 * 32 * 37), (3, 3 * 32 * 5), (5, 5 * 32 * 29), (8, 8 * 32 * 301), (16, 16 * 32 * 11),
          (7, 7 * 32)]


def _run(fc, calls, seed, dtype, phases=None):
    for k in range(calls):
        x = outlier_gaussian(fc.P, fc.n, seed=seed, call=k, dtype=dtype) if k % 2 else \
            gaussian(fc.P, fc.n, seed=seed, call=k, dtype=dtype)
        fc.call(x, phase=phases[k] if phases else 0)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("P,n", SHAPES)
def test_fused_sequences(oracle, P, n, dtype):
    fc = FullCompare(oracle, P, n, dtype, fused=True)
    try:
        _run(fc, 6, 40 + P, dtype, phases=[0, 0, 1, 1, 0, 1])
    finally:
        fc.close()


@pytest.mark.parametrize("variant", [OWNER_SUM, SENDER_EF, OWNER_SUM | SENDER_EF, FP16_SCALE,
                                     FP16_SCALE | SENDER_EF, FP16_SCALE | OWNER_SUM],
                         ids=["owner_sum", "sender_ef", "both", "fp16_scale", "fp16_ef", "fp16_owner_sum"])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_fused_variants(oracle, variant, dtype):
    P, n = 4, 4 * 32 * 29
    fc = FullCompare(oracle, P, n, dtype, variant=variant, fused=True)
    try:
        _run(fc, 5, 41, dtype, phases=[0, 1, 0, 1, 0])
    finally:
        fc.close()


@pytest.mark.parametrize("fp16", [False, True], ids=["pow2", "fp16_scale"])
@pytest.mark.parametrize("P", [2, 5])
@pytest.mark.parametrize("G", [16, 64, 128])
def test_fused_groups(oracle, G, P, fp16):
    n = P * G * 14  # a multiple of 32 at every G and P; n/8 not a multiple of 32 chunks
    for dtype in ("bf16", "fp32"):
        fc = FullCompare(oracle, P, n, dtype, group=G, variant=FP16_SCALE if fp16 else 0, fused=True)
        try:
            _run(fc, 4, 42 + G, dtype, phases=[0, 1, 1, 0])
        finally:
            fc.close()


@pytest.mark.parametrize("kind", ["zeros", "subnormal", "huge", "tiny_normal", "identical", "cancel", "ties",
                                  "one_outlier"])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_fused_edge_values(oracle, kind, dtype):
    P, n = 4, 4 * 32 * 45
    fc = FullCompare(oracle, P, n, dtype, fused=True)
    try:
        for k in range(3):
            x = _edge_inputs(P, n, kind) * np.float32(1 + k / 8)
            fc.call(bf16_bits(x) if dtype == "bf16" else x)
    finally:
        fc.close()


@pytest.mark.parametrize("kind", ["saturating", "tiny", "subnormal", "ties", "near_ties", "boundary", "zeros"])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_fused_fp16_scale_edge_values(oracle, kind, dtype):
    P, G = 4, 32
    n = P * G * 24
    fc = FullCompare(oracle, P, n, dtype, params=Params(enable=kind != "saturating"), variant=FP16_SCALE,
                     fused=True)
    try:
        for c in range(3):
            x = _fp16_edge(kind, P, n, G) * np.float32(1 + c / 16)
            fc.call(bf16_bits(x) if dtype == "bf16" else x)
    finally:
        fc.close()


@pytest.mark.parametrize("params", [
    Params(lam=0.25, beta_fast=0.3, beta_slow=0.95),
    Params(lam=1.0, beta_fast=0.0, beta_slow=0.875),
    Params(enable=False),
], ids=["asymmetric", "error_feedback", "off"])
def test_fused_parameters(oracle, params):
    P, n = 4, 4 * 32 * 257
    fc = FullCompare(oracle, P, n, "bf16", params, fused=True)
    try:
        _run(fc, 5, 43, "bf16")
    finally:
        fc.close()


def test_fused_out_of_place(oracle):
    P, n = 8, 8 * 32 * 77
    for dtype in ("bf16", "fp32"):
        fc = FullCompare(oracle, P, n, dtype, fused=True)
        try:
            for k in range(3):
                fc.call(gaussian(P, n, seed=44, call=k, dtype=dtype), out_of_place=True)
        finally:
            fc.close()


@pytest.mark.parametrize("P", list(range(2, 17)))
def test_fused_smallest_tensor(oracle, P):
    n = P * 32  # one group per owner: one warp, 4P of its lanes in the range
    fc = FullCompare(oracle, P, n, "bf16", fused=True)
    try:
        _run(fc, 3, 45 + P, "bf16")
    finally:
        fc.close()


def _snapshot(h, P, variant):
    snap = [h.get_wire(1, r) for r in range(P)] + [h.get_wire(2)]
    snap += [h.get_state(ph) for ph in (0, 1)]
    if variant & SENDER_EF:
        snap += [(h.get_sender_state(ph, r),) for ph in (0, 1) for r in range(P)]
    return snap


@pytest.mark.parametrize("variant", [0, OWNER_SUM | SENDER_EF, FP16_SCALE], ids=["default", "both", "fp16_scale"])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("n", [1 << 18, 8 * 32 * 4099], ids=["2e18", "above_2e20"])
def test_paths_identical(n, dtype, variant):
    """At sizes past the oracle's reach, the one-kernel path and the three
    kernels give the same bytes everywhere, call after call."""
    import torch
    from bit_error_compensated_rank_b200 import echo
    from bit_error_compensated_rank_b200 import workloads as wl
    P = 8
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    hs = [echo.Echo(P, n, echo.ECHO_BF16 if dtype == "bf16" else echo.ECHO_FP32) for _ in range(2)]
    try:
        for h, limit in zip(hs, (n, 0)):
            h.set_fused_limit(limit)
            h.set_params(0.3, 0.95, 0.25, 1)
            if variant:
                h.set_variant(variant)
        for c, ph in enumerate([0, 1, 0, 0]):
            outs = []
            for h in hs:
                x = [torch.empty(n, device="cuda", dtype=tdt) for _ in range(P)]
                for r in range(P):
                    wl.torch_outlier_gaussian_(x[r], seed=46, call=c, rank=r)
                h.allreduce(x, ph)
                outs.append(x)
            torch.cuda.synchronize()
            for r in range(P):
                assert torch.equal(outs[0][r].view(torch.int16 if dtype == "bf16" else torch.int32),
                                   outs[1][r].view(torch.int16 if dtype == "bf16" else torch.int32)), r
            for a, b in zip(_snapshot(hs[0], P, variant), _snapshot(hs[1], P, variant)):
                for u, v in zip(a, b):
                    assert_same_bits(u, v, "one kernel against three")
            assert all(h.device_status() == 0 for h in hs)
    finally:
        for h in hs:
            h.close()


def test_default_limit_and_timing():
    """Calls up to 2^20 elements per rank run as one kernel by default (timed
    as kernel 1, kernels 2 and 3 at zero); larger calls run the three."""
    import torch
    from bit_error_compensated_rank_b200 import echo
    P = 4
    for n, fused in [(1 << 20, True), ((1 << 20) + P * 32 * 16, False)]:
        h = echo.Echo(P, n)
        try:
            assert h.fused_limit() == 1 << 20
            x = [torch.randn(n, device="cuda").to(torch.bfloat16) for _ in range(P)]
            h.set_timing(True)
            h.allreduce(x)
            ms = h.last_kernel_ms()
            assert ms[0] > 0
            assert (ms[1] == 0 and ms[2] == 0) if fused else (ms[1] > 0 and ms[2] > 0), (n, ms)
        finally:
            h.close()


def test_fused_host_end_to_end(oracle):
    """echo_allreduce_host on a small tensor: pinned host partials in, the
    host result out, through the one-kernel path."""
    import torch
    from bit_error_compensated_rank_b200 import echo
    P, n = 4, 4 * 32 * 300
    h = echo.Echo(P, n)
    try:
        assert n <= h.fused_limit()
        f = np.zeros(n, np.float32)
        s = np.zeros(n, np.float32)
        for c in range(3):
            x = outlier_gaussian(P, n, seed=47, call=c)
            host_in = [torch.from_numpy(x[r].view(np.int16)).view(torch.bfloat16).pin_memory()
                       for r in range(P)]
            host_out = torch.empty(n, dtype=torch.bfloat16).pin_memory()
            h.allreduce_host(host_in, host_out)
            ref = oracle.allreduce(x, f, s, Params())
            assert_same_bits(host_out.view(torch.int16).numpy().view(np.uint16), ref["out"],
                             f"host output call {c}")
        gf, gs = h.get_state(0)
        assert_same_bits(gf, f, "fast estimate")
        assert_same_bits(gs, s, "slow estimate")
    finally:
        h.close()
