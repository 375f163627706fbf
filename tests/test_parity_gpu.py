"""CUDA path against the CPU oracle, bit for bit, on problems small enough to
compare in full (several warp steps, CTAs and grid-stride rounds, ragged
tails), through the C ABI."""
import os
import subprocess
import sys

import numpy as np
import pytest

from bit_error_compensated_rank_b200.workloads import bf16_bits, gaussian, outlier_gaussian, rng
from bit_error_compensated_rank_b200 import workloads as wl
from gpu_harness import FullCompare, SampledCompare, assert_same_bits, from_device, to_device
from oracle.oracle import Params

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# n = P * 32 * k with k chosen so the chunk count (n/8) is not a multiple of a
# warp step (32 chunks) or of a CTA step (256 chunks): ragged tails everywhere.
SHAPES = [(2, 2 * 32 * 37), (3, 3 * 32 * 41), (4, 4 * 32 * 64), (5, 5 * 32 * 29),
          (8, 8 * 32 * 3001), (16, 16 * 32 * 101), (7, 7 * 32)]


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("P,n", SHAPES)
def test_sequence_both_phases(oracle, P, n, dtype):
    fc = FullCompare(oracle, P, n, dtype)
    try:
        phases = [0, 0, 0, 1, 1, 0]
        for k, ph in enumerate(phases):
            x = outlier_gaussian(P, n, seed=P, call=k, dtype=dtype) if k % 2 else \
                gaussian(P, n, seed=P, call=k, dtype=dtype)
            fc.call(x, phase=ph)
    finally:
        fc.close()


@pytest.mark.parametrize("params", [
    Params(lam=0.25, beta_fast=0.3, beta_slow=0.95),
    Params(lam=1.0, beta_fast=0.0, beta_slow=0.875),
    Params(lam=0.5, beta_fast=0.5, beta_slow=0.875, enable=False),
], ids=["asymmetric", "error_feedback", "off"])
def test_parameters(oracle, params):
    P, n = 4, 4 * 32 * 257
    fc = FullCompare(oracle, P, n, "bf16", params)
    try:
        for k in range(5):
            fc.call(gaussian(P, n, seed=21, call=k), phase=0)
    finally:
        fc.close()


def test_out_of_place(oracle):
    P, n = 8, 8 * 32 * 77
    for dtype in ("bf16", "fp32"):
        fc = FullCompare(oracle, P, n, dtype)
        try:
            for k in range(3):
                fc.call(gaussian(P, n, seed=3, call=k, dtype=dtype), out_of_place=True)
        finally:
            fc.close()


def _edge_inputs(P, n, kind):
    g = rng(17, P, len(kind))
    if kind == "zeros":
        return np.zeros((P, n), np.float32)
    if kind == "subnormal":
        return (g.integers(-2 ** 20, 2 ** 20, (P, n)) * 2.0 ** -149).astype(np.float32)
    if kind == "huge":
        return (g.standard_normal((P, n)) * 2.0 ** 100).astype(np.float32)
    if kind == "tiny_normal":
        return (g.standard_normal((P, n)) * 2.0 ** -120).astype(np.float32)
    if kind == "identical":
        return np.repeat(g.standard_normal((1, n)).astype(np.float32), P, axis=0)
    if kind == "cancel":
        x = g.standard_normal((P, n)).astype(np.float32)
        x[1::2] = -x[0::2][: x[1::2].shape[0]]
        return x
    if kind == "ties":
        k = g.integers(-7, 7, (P, n)) + 0.5
        k[:, ::32] = 7
        return (k * 2.0 ** g.integers(-20, 20, (P, 1))).astype(np.float32)
    if kind == "one_outlier":
        x = g.standard_normal((P, n)).astype(np.float32)
        x[:, 5::32] *= 1000
        return x
    raise ValueError(kind)


@pytest.mark.parametrize("kind", ["zeros", "subnormal", "huge", "tiny_normal", "identical",
                                  "cancel", "ties", "one_outlier"])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_edge_values(oracle, kind, dtype):
    P, n = 4, 4 * 32 * 45
    fc = FullCompare(oracle, P, n, dtype)
    try:
        for k in range(3):
            x = _edge_inputs(P, n, kind)
            if k:
                x = x * np.float32(1 + k / 8)
            fc.call(bf16_bits(x) if dtype == "bf16" else x)
    finally:
        fc.close()


@pytest.mark.parametrize("P", list(range(2, 17)))
def test_smallest_tensor(oracle, P):
    n = P * 32  # one group per owner
    fc = FullCompare(oracle, P, n, "bf16")
    try:
        for k in range(3):
            fc.call(gaussian(P, n, seed=P, call=k))
    finally:
        fc.close()


def test_state_set_get_reset(oracle):
    from bit_error_compensated_rank_b200 import echo
    P, n = 4, 4 * 32 * 33
    fc = FullCompare(oracle, P, n, "bf16")
    try:
        g = rng(5, 5)
        for ph in (0, 1):
            f = (g.standard_normal(n) * 0.05).astype(np.float32)
            s = (g.standard_normal(n) * 0.05).astype(np.float32)
            fc.h.set_state(ph, f, s)
            gf, gs = fc.h.get_state(ph)
            assert_same_bits(gf, f, "set/get f")
            assert_same_bits(gs, s, "set/get s")
            fc.state[ph] = (f.copy(), s.copy())
        for k in range(3):
            fc.call(gaussian(P, n, seed=6, call=k), phase=k % 2)
        fc.h.reset(1)
        gf, gs = fc.h.get_state(0)
        assert not gf.any() and not gs.any()
        gf1, _ = fc.h.get_state(1)
        assert_same_bits(gf1, fc.state[1][0], "bwd state kept by a fwd reset")
        fc.state[0] = (np.zeros(n, np.float32), np.zeros(n, np.float32))
        fc.call(gaussian(P, n, seed=6, call=9), phase=0)
        st = fc.h.stats()
        mb = echo.echo_model_bytes(P, n, echo.ECHO_BF16, True)
        assert st["calls"] == 4
        assert st["link_bytes"] == 4 * mb["link"]
        assert st["model_hbm_bytes"] == 4 * mb["total"]
    finally:
        fc.close()


def test_timing_events():
    import torch
    from bit_error_compensated_rank_b200 import echo
    P, n = 8, 8 * 32 * 4096
    h = echo.Echo(P, n)
    h.set_fused_limit(0)  # the three kernels, each timed
    try:
        x = [torch.randn(n, device="cuda").to(torch.bfloat16) for _ in range(P)]
        h.set_timing(True)
        h.allreduce(x)
        ms = h.last_kernel_ms()
        assert len(ms) == 3 and all(m > 0 for m in ms)
        h.set_timing(False)
        h.allreduce(x)
        with pytest.raises(echo.EchoError):
            h.last_kernel_ms()
    finally:
        h.close()


def test_rejects_bad_buffers_without_launching():
    import torch
    from bit_error_compensated_rank_b200 import echo
    P, n = 4, 4 * 32 * 16
    h = echo.Echo(P, n)
    try:
        x = [torch.zeros(n, device="cuda", dtype=torch.bfloat16) for _ in range(P)]
        h.allreduce(x)
        big = torch.zeros(P * n + 8, device="cuda", dtype=torch.bfloat16)
        cases = {
            "misaligned": [x[0].data_ptr() + 2] + [t.data_ptr() for t in x[1:]],
            "overlap": [big.data_ptr() + r * (n - 8) * 2 for r in range(P)],
            "duplicate": [x[0].data_ptr()] * P,
            "host": [np.zeros(n, np.uint16).ctypes.data // 16 * 16 + 16] + [t.data_ptr() for t in x[1:]],
            "null": [0] + [t.data_ptr() for t in x[1:]],
        }
        for name, ptrs in cases.items():
            with pytest.raises(echo.EchoError) as ei:
                echo.echo_allreduce(h.h, ptrs, 0, 0)
            assert ei.value.code == echo.ECHO_ERR_INVALID, name
        with pytest.raises(echo.EchoError):
            echo.echo_allreduce(h.h, [t.data_ptr() for t in x], 2, 0)
        with pytest.raises(echo.EchoError):
            h.set_params(1.0, 0.5, 0.5, True)
        # the torch wrapper checks what the C ABI cannot see: count, size, dtype, layout
        wrapper_cases = {
            "count": x[:-1],
            "short": x[:-1] + [torch.zeros(n - 32, device="cuda", dtype=torch.bfloat16)],
            "dtype": x[:-1] + [torch.zeros(n, device="cuda", dtype=torch.float32)],
            "strided": x[:-1] + [torch.zeros(2 * n, device="cuda", dtype=torch.bfloat16)[::2]],
            "cpu": x[:-1] + [torch.zeros(n, dtype=torch.bfloat16)],
        }
        for name, tensors in wrapper_cases.items():
            with pytest.raises(echo.EchoError) as ei:
                h.allreduce(tensors)
            assert ei.value.code == echo.ECHO_ERR_INVALID, name
        assert h.stats()["calls"] == 1
        torch.cuda.synchronize()
    finally:
        h.close()


def test_injected_launch_failure():
    code = (
        "import os; os.environ['ECHO_FAULT'] = 'launch'\n"
        "import torch\n"
        "from bit_error_compensated_rank_b200 import echo as e\n"
        "h = e.Echo(2, 64)\n"
        "x = [torch.zeros(64, device='cuda', dtype=torch.bfloat16) for _ in range(2)]\n"
        "try:\n"
        "    h.allreduce(x)\n"
        "    raise SystemExit('no error')\n"
        "except e.EchoError as err:\n"
        "    assert err.code == e.ECHO_ERR_CUDA and 'injected' in str(err), err\n"
        "assert h.stats()['calls'] == 0\n"
        "h.close()\n"
    )
    res = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr + res.stdout


def test_bounded_waits_report_timeouts():
    """With ECHO_FAULT=stall the kernels issue no loads, so the first wait of
    every CTA runs out after its (short) bound: each kernel records its bit in
    the device status word and returns, and the context stays usable."""
    code = (
        "import os; os.environ['ECHO_FAULT'] = 'stall'\n"
        "import torch\n"
        "from bit_error_compensated_rank_b200 import echo as e\n"
        "h = e.Echo(4, 4 * 32 * 1000)\n"
        "x = [torch.zeros(4 * 32 * 1000, device='cuda', dtype=torch.bfloat16) for _ in range(4)]\n"
        "h.allreduce(x)\n"
        "torch.cuda.synchronize()\n"
        "assert h.device_status() == 7, h.device_status()\n"
        "assert h.device_status(clear=True) == 7\n"
        "assert h.device_status() == 0\n"
        "y = torch.ones(1024, device='cuda') * 2\n"
        "assert float(y.sum()) == 2048.0\n"
        "h.close()\n"
    )
    res = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                         timeout=120)
    assert res.returncode == 0, res.stderr + res.stdout


def test_no_timeouts_in_normal_calls(oracle):
    P, n = 8, 8 * 32 * 5000
    fc = FullCompare(oracle, P, n, "bf16")
    try:
        for k in range(2):
            fc.call(gaussian(P, n, seed=31, call=k))
        assert fc.h.device_status() == 0
    finally:
        fc.close()


def test_host_end_to_end(oracle):
    """Host buffers in, host result out (one piece: the host path moves
    pieces of 2^25 elements; the binary32 case below spans two)."""
    import torch
    from bit_error_compensated_rank_b200 import echo
    P, n = 4, 4 * 32 * 80000  # 10.24 M elements per rank
    h = echo.Echo(P, n)
    try:
        f = np.zeros(n, np.float32)
        s = np.zeros(n, np.float32)
        for k in range(2):
            x = gaussian(P, n, seed=8, call=k)
            host_in = [torch.from_numpy(x[r].view(np.int16)).view(torch.bfloat16).pin_memory()
                       for r in range(P)]
            host_out = torch.empty(n, dtype=torch.bfloat16).pin_memory()
            h.allreduce_host(host_in, host_out)
            ref = oracle.allreduce(x, f, s, Params())
            assert_same_bits(host_out.view(torch.int16).numpy().view(np.uint16), ref["out"], "host result")
            gf, gs = h.get_state(0)
            assert_same_bits(gf, f, "fast estimate")
            assert_same_bits(gs, s, "slow estimate")
    finally:
        h.close()


def test_largest_tensor_sampled(oracle):
    """More than 2^31 elements per rank (P = 2, n = 3 * 2^30 + 64, ragged
    against every tile length): byte offsets past 2^32 in the partials, the
    state and the wire, 32-bit chunk indices near their top. About 70 GB of
    device memory; sampled blocks at both ends, the segment boundary and
    random places, compared exactly after each of two calls."""
    import torch
    torch.cuda.empty_cache()
    P, n = 2, 3 * (1 << 30) + 64
    sc = SampledCompare(oracle, P, n, "bf16", block_groups=32)
    try:
        bufs = [torch.empty(n, device="cuda", dtype=torch.bfloat16) for _ in range(P)]
        for k in range(2):
            for r in range(P):
                wl.torch_outlier_gaussian_(bufs[r], seed=21, call=k, rank=r)
            sc.call(bufs, phase=k)
    finally:
        sc.close()
        del bufs
        torch.cuda.empty_cache()


@pytest.mark.parametrize("fused", [False, True], ids=["three_kernels", "one_kernel"])
def test_cuda_graph_replay(oracle, fused):
    """Calls captured once in a CUDA graph and replayed: every replay is a
    correct call (the kernels read their launch shape from the arguments, and
    the state moves on device), bit for bit the oracle's sequence."""
    import torch
    from bit_error_compensated_rank_b200 import echo
    P, n, per_graph, replays = 8, 8 * 32 * 1024, 3, 3
    h = echo.Echo(P, n)
    h.set_fused_limit(n if fused else 0)
    try:
        x = gaussian(P, n, seed=95, call=0)
        send = to_device(x)
        recv = [torch.empty_like(t) for t in send]
        stream = torch.cuda.Stream()
        with torch.cuda.stream(stream):
            h.allreduce_out(send, recv, 0, stream)  # warm-up outside the capture
        torch.cuda.synchronize()
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


def test_host_end_to_end_fp32_backward(oracle):
    """The host path with binary32 partials, in the backward phase, over a
    ragged last piece; the forward state stays untouched."""
    import torch
    from bit_error_compensated_rank_b200 import echo
    P, n = 2, 2 * 32 * ((1 << 19) + 1)  # 2^25 + 64 elements per rank: a full piece and a ragged one
    h = echo.Echo(P, n, echo.ECHO_FP32)
    try:
        f = np.zeros(n, np.float32)
        s = np.zeros(n, np.float32)
        for k in range(2):
            x = gaussian(P, n, seed=18, call=k, dtype="fp32")
            host_in = [torch.from_numpy(np.ascontiguousarray(x[r])).pin_memory() for r in range(P)]
            host_out = torch.empty(n, dtype=torch.float32).pin_memory()
            h.allreduce_host(host_in, host_out, echo.ECHO_BWD)
            ref = oracle.allreduce(x, f, s, Params())
            assert_same_bits(host_out.numpy(), ref["out"], "host result")
            gf, gs = h.get_state(echo.ECHO_BWD)
            assert_same_bits(gf, f, "fast estimate")
            assert_same_bits(gs, s, "slow estimate")
            ff, fs = h.get_state(echo.ECHO_FWD)
            assert not ff.any() and not fs.any()
    finally:
        h.close()


@pytest.mark.parametrize("variant", [0, 4], ids=["default", "fp16_scale"])
@pytest.mark.parametrize("P", [11, 12, 13, 16])
def test_many_ranks_full_tiles(oracle, P, variant):
    """From P = 11 on, kernel 2's stages no longer fit two full tiles, so the
    tile halves and the ring deepens to three stages. About 4 Mi elements per
    rank give full-size tiles, several turns of the ring per CTA and a ragged
    last tile; compared in full over two calls, the second corrected by the
    state the first left."""
    n = P * 32 * ((1 << 22) // (P * 32) + 3)
    fc = FullCompare(oracle, P, n, "bf16", variant=variant)
    try:
        for k in range(2):
            fc.call(outlier_gaussian(P, n, seed=60 + P, call=k), phase=0)
    finally:
        fc.close()
