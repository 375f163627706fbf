"""The all-reduce entry point that allocates nothing, checked against the
ordinary one.

echo_allreduce_static exists for callers that cannot allocate device memory
when they reduce: a serving process that reserved all of HBM for its own pool
at start-up, a plugin inside a host application that owns every allocation,
or a latency-critical path where a cudaMalloc (which can synchronise the
device) is not acceptable. Its wire buffers live in a fixed array compiled
into the library; the caller passes the rank buffers and the compensator
state.

The tests call it through the C ABI. Two compare it over two calls in a row
(so the state carried from the first call is checked too): one with
echo_allreduce on a handle, one with the CPU oracle directly. Outputs and
state must agree bit for bit, which is the tolerance of every parity test
here. Another checks what the entry point is for: once it is set up, calls
change neither the device's free memory nor torch's allocations. Further
tests cover its argument rejections (nothing enqueued) and its status word.
This file sorts last so a run that stops at the first failure has already
run everything else; it also passes alone in a fresh process.
"""
import gc
import os
import subprocess
import sys

import numpy as np
import pytest

from bit_error_compensated_rank_b200.workloads import bf16_bits, outlier_gaussian

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _device_copies(x):
    import torch
    if x.dtype == np.uint16:
        base = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)
    else:
        base = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    return [base[r].clone() for r in range(x.shape[0])]


def _bits(t):
    import torch
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy().view(np.uint32)


# n <= 2^20 runs as one kernel, larger n as the three kernels, on both sides
@pytest.mark.parametrize("P,n,dtype", [(8, 8 * 32 * 4096, "bf16"), (4, 4 * 32 * 2003, "fp32"),
                                       (4, 4 * 32 * 8200, "bf16")])
def test_static_entry_point_matches_handle(P, n, dtype):
    import torch
    from bit_error_compensated_rank_b200 import echo

    code = echo.ECHO_BF16 if dtype == "bf16" else echo.ECHO_FP32
    h = echo.Echo(P, n, code)
    f = torch.zeros(n, dtype=torch.float32, device="cuda")
    s = torch.zeros(n, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    try:
        for call in range(2):
            x = outlier_gaussian(P, n, seed=77, call=call, dtype="fp32")
            if dtype == "bf16":
                x = bf16_bits(x)
            ref = _device_copies(x)
            got = _device_copies(x)
            h.allreduce(ref, echo.ECHO_FWD)
            echo.echo_allreduce_static(P, n, code, [t.data_ptr() for t in got], f.data_ptr(),
                                       s.data_ptr(), 0.5, 0.875, 0.5, True, stream)
            torch.cuda.synchronize()
            for r in range(P):
                assert (_bits(got[r]) == _bits(ref[r])).all(), (call, r)
            hf, hs = h.get_state(echo.ECHO_FWD)
            assert (f.cpu().numpy().view(np.uint32) == hf.view(np.uint32)).all(), call
            assert (s.cpu().numpy().view(np.uint32) == hs.view(np.uint32)).all(), call
    finally:
        h.close()


def test_static_entry_point_rejects_sizes_beyond_its_scratch():
    import torch
    from bit_error_compensated_rank_b200 import echo

    P, n = 8, 8 * 32 * 65536  # 16.8 M elements per rank: about 80 MiB of wire
    bufs = [torch.zeros(n, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    f = torch.zeros(n, dtype=torch.float32, device="cuda")
    s = torch.zeros(n, dtype=torch.float32, device="cuda")
    with pytest.raises(echo.EchoError) as ei:
        echo.echo_allreduce_static(P, n, echo.ECHO_BF16, [t.data_ptr() for t in bufs], f.data_ptr(),
                                   s.data_ptr())
    assert ei.value.code == echo.ECHO_ERR_UNSUPPORTED
    assert "static scratch" in str(ei.value)
    torch.cuda.synchronize()
    assert not any(bool(t.any()) for t in bufs)  # nothing was enqueued


@pytest.mark.parametrize("P,n,dtype", [(4, 4 * 32 * 96, "bf16"), (3, 3 * 32 * 40, "fp32"),
                                       (2, 2 * 32 * 16400, "bf16")])
def test_static_entry_point_matches_oracle(oracle, P, n, dtype):
    import torch
    from bit_error_compensated_rank_b200 import echo
    from oracle.oracle import Params

    code = echo.ECHO_BF16 if dtype == "bf16" else echo.ECHO_FP32
    f = torch.zeros(n, dtype=torch.float32, device="cuda")
    s = torch.zeros(n, dtype=torch.float32, device="cuda")
    fo = np.zeros(n, np.float32)
    so = np.zeros(n, np.float32)
    prm = Params(lam=0.25, beta_fast=0.3, beta_slow=0.95)
    for call in range(2):
        x = outlier_gaussian(P, n, seed=78, call=call, dtype="fp32")
        if dtype == "bf16":
            x = bf16_bits(x)
        got = _device_copies(x)
        echo.echo_allreduce_static(P, n, code, [t.data_ptr() for t in got], f.data_ptr(),
                                   s.data_ptr(), prm.beta_fast, prm.beta_slow, prm.lam, True,
                                   torch.cuda.current_stream().cuda_stream)
        torch.cuda.synchronize()
        ref = oracle.allreduce(x, fo, so, prm, want_wire=False)
        want = ref["out"].view(np.uint16 if dtype == "bf16" else np.uint32)
        for r in range(P):
            assert (_bits(got[r]) == want).all(), (call, r)
        assert (f.cpu().numpy().view(np.uint32) == fo.view(np.uint32)).all(), call
        assert (s.cpu().numpy().view(np.uint32) == so.view(np.uint32)).all(), call
    assert echo.echo_static_status() == 0


@pytest.mark.parametrize("n", [8 * 32 * 4096, 8 * 32 * 4200], ids=["one_kernel", "three_kernels"])
def test_static_calls_allocate_nothing(n):
    """After the set-up call, further calls leave the device's free memory
    and torch's allocation counters exactly as they were."""
    import torch
    from bit_error_compensated_rank_b200 import echo

    P = 8
    bufs = [torch.randn(n, device="cuda").to(torch.bfloat16) for _ in range(P)]
    f = torch.zeros(n, dtype=torch.float32, device="cuda")
    s = torch.zeros(n, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    ptrs = [t.data_ptr() for t in bufs]

    def call():
        echo.echo_allreduce_static(P, n, echo.ECHO_BF16, ptrs, f.data_ptr(), s.data_ptr(),
                                   stream=stream)

    call()  # set-up (and first launch of each kernel) happens here
    torch.cuda.synchronize()
    # Tensors that earlier tests left in reference cycles would otherwise be
    # freed whenever the garbage collector runs, moving torch's counters.
    gc.collect()
    gc.disable()
    try:
        free0, _ = torch.cuda.mem_get_info()
        alloc0 = torch.cuda.memory_allocated()
        reserved0 = torch.cuda.memory_reserved()
        for _ in range(5):
            call()
        torch.cuda.synchronize()
        free1, _ = torch.cuda.mem_get_info()
        assert free1 == free0, (free0, free1)
        assert torch.cuda.memory_allocated() == alloc0
        assert torch.cuda.memory_reserved() == reserved0
    finally:
        gc.enable()
    assert echo.echo_static_status() == 0


def test_static_rejects_bad_pointers_with_nothing_enqueued():
    """Each pointer error returns ECHO_ERR_INVALID before anything reaches
    the stream: the rank buffers and the state keep their values."""
    import ctypes

    import torch
    from bit_error_compensated_rank_b200 import echo

    P, n = 4, 4 * 32 * 64
    nbytes = n * 2
    bufs = [torch.randn(n, device="cuda").to(torch.bfloat16) for _ in range(P)]
    f = torch.full((n,), 0.25, dtype=torch.float32, device="cuda")
    s = torch.full((n,), 0.5, dtype=torch.float32, device="cuda")
    big = torch.zeros(2 * n, dtype=torch.bfloat16, device="cuda")
    before = [t.clone() for t in bufs]
    host = (ctypes.c_uint8 * nbytes)()
    host_ptr = (ctypes.addressof(host) + 15) // 16 * 16
    good = [t.data_ptr() for t in bufs]
    fp, sp = f.data_ptr(), s.data_ptr()
    cases = [
        ("NULL rank array", None, fp, sp, 1, "NULL"),
        ("NULL rank pointer", good[:2] + [0] + good[3:], fp, sp, 1, "NULL"),
        ("misaligned", [good[0] + 2] + good[1:], fp, sp, 1, "aligned"),
        ("host memory", [host_ptr] + good[1:], fp, sp, 1, "device"),
        ("overlapping ranks", [big.data_ptr(), big.data_ptr() + nbytes // 2] + good[2:], fp, sp, 1,
         "overlap"),
        ("NULL state", good, 0, sp, 1, "NULL"),
        ("state arrays overlap", good, fp, fp + 64, 1, "overlap"),
        ("state overlaps a rank", good, good[1], sp, 1, "overlap"),
    ]
    for what, ptrs, fpp, spp, en, words in cases:
        arr = None if ptrs is None else echo._ptr_array(ptrs)
        rc = echo._lib.echo_allreduce_static(P, n, echo.ECHO_BF16, arr, fpp, spp, 0.5, 0.875, 0.5, en,
                                             None)
        assert rc == echo.ECHO_ERR_INVALID, (what, rc, echo.echo_last_error())
        assert words in echo.echo_last_error(), (what, echo.echo_last_error())
    torch.cuda.synchronize()
    for a, b in zip(bufs, before):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert bool((f == 0.25).all()) and bool((s == 0.5).all())
    assert echo.echo_static_status() == 0


def test_static_status_reports_timeouts():
    """With ECHO_FAULT=stall the kernels issue no loads, so every CTA's first
    wait runs out after its short bound; each kernel records its bit in the
    static status word, which stays set until it is cleared, and the
    context stays usable."""
    code = (
        "import os; os.environ['ECHO_FAULT'] = 'stall'\n"
        "import torch\n"
        "from bit_error_compensated_rank_b200 import echo as e\n"
        "assert e.echo_static_status() == 0\n"
        "P, n = 4, 4 * 32 * 1000\n"
        "x = [torch.zeros(n, device='cuda', dtype=torch.bfloat16) for _ in range(P)]\n"
        "f = torch.zeros(n, device='cuda'); s = torch.zeros(n, device='cuda')\n"
        "e.echo_allreduce_static(P, n, e.ECHO_BF16, [t.data_ptr() for t in x], f.data_ptr(), s.data_ptr())\n"
        "torch.cuda.synchronize()\n"
        "assert e.echo_static_status() == 7, e.echo_static_status()\n"
        "assert e.echo_static_status(clear=True) == 7\n"
        "assert e.echo_static_status() == 0\n"
        "y = torch.ones(1024, device='cuda') * 2\n"
        "assert float(y.sum()) == 2048.0\n"
    )
    res = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                         timeout=120)
    assert res.returncode == 0, res.stderr + res.stdout
