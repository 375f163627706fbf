"""The all-reduce entry point that allocates nothing, checked against the
ordinary one.

echo_allreduce_static exists for callers that cannot allocate device memory
when they reduce: a serving process that reserved all of HBM for its own pool
at start-up, a plugin inside a host application that owns every allocation,
or a latency-critical path where a cudaMalloc (which can synchronise the
device) is not acceptable. Its wire buffers live in a fixed array compiled
into the library; the caller passes the rank buffers and the compensator
state.

Each test compares it, through the C ABI, with echo_allreduce on a handle over
two calls in a row (so the state carried from the first call is checked too):
outputs and state must agree bit for bit, which is the tolerance of every
parity test here. This file sorts last so a run that stops at the first
failure has already run everything else; it also passes alone in a fresh
process.
"""
import numpy as np
import pytest

from bit_error_compensated_rank_b200.workloads import bf16_bits, outlier_gaussian

pytestmark = pytest.mark.gpu


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


@pytest.mark.parametrize("P,n,dtype", [(8, 8 * 32 * 4096, "bf16"), (4, 4 * 32 * 2003, "fp32")])
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
