"""The one-launch path (ECHO_PATH_FUSED, and ECHO_PATH_AUTO for small calls)
against the oracle, bit for bit: the same three steps in one cooperative
launch with a grid-wide barrier between them.

Compared after every call: both wires, every rank's output, both phases'
estimates and every rank's sender error, for every variant, group size and
scale format; plus repeated CUDA-graph replays (the barrier must return to its
rest state after every launch), the injected barrier timeout, and the choice
the automatic path makes."""
import os
import subprocess
import sys

import numpy as np
import pytest

from bit_error_compensated_rank_b200.workloads import gaussian, outlier_gaussian
from gpu_harness import FullCompare, assert_same_bits, from_device, to_device
from oracle.oracle import FP16_SCALE, OWNER_SUM, SENDER_EF, Params

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("P,n", [(2, 4096), (2, 2 * 32), (3, 3 * 32 * 7), (5, 5 * 32 * 33),
                                 (8, 8 * 32 * 301), (16, 16 * 32 * 17), (4, 4 * 32 * 4096)])
def test_fused_sequences(oracle, P, n, dtype):
    fc = FullCompare(oracle, P, n, dtype, path="fused")
    try:
        for k, ph in enumerate([0, 0, 1, 0, 1, 1]):
            fc.call(outlier_gaussian(P, n, seed=90 + P, call=k, dtype=dtype), phase=ph)
    finally:
        fc.close()


@pytest.mark.parametrize("variant", [OWNER_SUM, SENDER_EF, OWNER_SUM | SENDER_EF, FP16_SCALE,
                                     FP16_SCALE | SENDER_EF | OWNER_SUM],
                         ids=["owner_sum", "sender_ef", "both", "fp16", "fp16_both"])
@pytest.mark.parametrize("G", [16, 32, 128])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_fused_variants(oracle, variant, G, dtype):
    P = 4
    n = P * G * 24
    fc = FullCompare(oracle, P, n, dtype, group=G, variant=variant, path="fused")
    try:
        for k in range(4):
            fc.call(outlier_gaussian(P, n, seed=91, call=k, dtype=dtype), phase=k & 1,
                    out_of_place=bool(k & 1))
    finally:
        fc.close()


def test_fused_compensation_off_and_parameters(oracle):
    P, n = 8, 8 * 32 * 64
    for params in (Params(enable=False), Params(lam=0.25, beta_fast=0.75, beta_slow=0.9375)):
        fc = FullCompare(oracle, P, n, "bf16", params=params, path="fused")
        try:
            for k in range(3):
                fc.call(gaussian(P, n, seed=92, call=k))
        finally:
            fc.close()


def test_paths_alternate_on_one_handle(oracle):
    """Switching between the paths keeps the state: both compute the same bits."""
    P, n = 4, 4 * 32 * 200
    fc = FullCompare(oracle, P, n, "bf16", variant=SENDER_EF)
    try:
        for k, path in enumerate([1, 2, 2, 1, 0, 2, 1]):
            fc.h.set_path(path)
            fc.call(gaussian(P, n, seed=93, call=k))
    finally:
        fc.close()


def test_fused_graph_replay(oracle):
    """Calls captured in a CUDA graph and replayed: the barrier words return
    to rest after each launch, so every replay is a correct call."""
    import torch
    from bit_error_compensated_rank_b200 import echo
    P, n, per_graph, replays = 4, 4 * 32 * 128, 3, 3
    h = echo.Echo(P, n)
    h.set_path(echo.ECHO_PATH_FUSED)
    try:
        x = gaussian(P, n, seed=94, call=0)
        send = to_device(x)
        recv = [torch.empty_like(t) for t in send]
        stream = torch.cuda.Stream()
        with torch.cuda.stream(stream):
            h.allreduce_out(send, recv, 0, stream)  # warm-up outside the capture
        torch.cuda.synchronize()
        h.reset()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for _ in range(per_graph):
                h.allreduce_out(send, recv, 0, stream)
        torch.cuda.synchronize()
        h.reset()
        f = np.zeros(n, np.float32)
        s = np.zeros(n, np.float32)
        for _ in range(replays):
            graph.replay()
            torch.cuda.synchronize()
            for _ in range(per_graph):
                ref = oracle.allreduce(x, f, s, Params())
            assert h.device_status(clear=True) == 0
            got = from_device(recv)
            for r in range(P):
                assert_same_bits(got[r], ref["out"], f"output rank {r}")
            gf, gs = h.get_state(0)
            assert_same_bits(gf, f, "fast estimate")
            assert_same_bits(gs, s, "slow estimate")
        del graph
    finally:
        h.close()


def test_fused_barrier_timeout_is_reported():
    """ECHO_FAULT=stall: the last CTA at the first barrier does not release
    the others, so their waits run out (bounded) and the status word gets
    ECHO_STATUS_TIMEOUT_FUSED; later one-launch calls do nothing until the
    word is cleared, after which calls are correct again."""
    code = r"""
import os
import numpy as np, torch
from bit_error_compensated_rank_b200 import echo as e
P, n = 4, 4 * 32 * 2000
h = e.Echo(P, n)
h.set_path(e.ECHO_PATH_FUSED)
x = [torch.ones(n, device="cuda", dtype=torch.bfloat16) for _ in range(P)]
os.environ["ECHO_FAULT"] = "stall"
h.allreduce(x)
torch.cuda.synchronize()
assert h.device_status() == e.ECHO_STATUS_TIMEOUT_FUSED, h.device_status()
del os.environ["ECHO_FAULT"]
y = [torch.ones(n, device="cuda", dtype=torch.bfloat16) for _ in range(P)]
h.allreduce(y)  # refused on the device while the bit is set: y untouched
torch.cuda.synchronize()
assert all(float(t.float().sum()) == n for t in y)
assert h.device_status(clear=True) == e.ECHO_STATUS_TIMEOUT_FUSED
h.reset()
h.allreduce(y)
torch.cuda.synchronize()
assert h.device_status() == 0
assert all(float(t.float().sum()) == P * n for t in y), [float(t.float().sum()) for t in y]
h.close()
print("ok")
"""
    res = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                         timeout=120)
    assert res.returncode == 0 and "ok" in res.stdout, res.stderr + res.stdout


def test_auto_path_choice():
    """The automatic path uses one launch up to 2^21 elements over all ranks:
    visible in the timing slots (the one-launch path puts the whole call in
    kernel 1's slot)."""
    import torch
    from bit_error_compensated_rank_b200 import echo
    for P, n, fused in [(8, 1 << 18, True), (8, 1 << 19, False), (2, 1 << 20, True)]:
        h = echo.Echo(P, n)
        try:
            x = [torch.randn(n, device="cuda").to(torch.bfloat16) for _ in range(P)]
            h.set_timing(True)
            h.allreduce(x)
            ms = h.last_kernel_ms()
            assert (ms[1] == 0 and ms[2] == 0) == fused, (P, n, ms)
        finally:
            h.close()


def test_fused_rejects_too_large():
    from bit_error_compensated_rank_b200 import echo
    h = echo.Echo(2, 1 << 30)
    try:
        with pytest.raises(echo.EchoError) as ei:
            h.set_path(echo.ECHO_PATH_FUSED)
        assert ei.value.code == echo.ECHO_ERR_UNSUPPORTED
    finally:
        h.close()
