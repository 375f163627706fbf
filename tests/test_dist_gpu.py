"""The all-reduce with one rank per handle (echo_dist_*), on one GPU: each
rank holds only its own partial and the state of the segment it owns, the
kernels store the wire straight into the other ranks' blocks (CUDA IPC
between processes, direct pointers between ranks of one process), and every
rank's result and owned state must equal the oracle's bit for bit, call after
call, for both phases, in place and out of place.

The stages are ordered on the GPU by the library's events and by host
barriers (gloo) between the stages; no kernel waits on another rank, so the
processes can share one GPU. One case runs the host-ordered form (stream
synchronised before each barrier) that the event ordering replaced."""
import pytest

from oracle.oracle import FP16_SCALE, OWNER_SUM, SENDER_EF

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world,nprocs,n,dtype,variant,group,sync", [
    (2, 2, 2 * 32 * 300, "bf16", 0, 32, False),
    (4, 4, 4 * 32 * 129, "fp32", 0, 32, False),
    (3, 3, 3 * 32 * 64, "bf16", OWNER_SUM | SENDER_EF, 32, False),
    (4, 4, 4 * 128 * 40, "bf16", FP16_SCALE, 128, False),
    (2, 2, 2 * 32 * 5000, "bf16", SENDER_EF, 16, False),
    (2, 2, 2 * 32 * 300, "bf16", 0, 32, True),
    (4, 2, 4 * 32 * 257, "bf16", 0, 32, False),
    (8, 2, 8 * 32 * 1024, "bf16", 0, 32, False),
], ids=["w2", "w4_fp32", "w3_both", "w4_fp16_g128", "w2_ef_g16", "w2_host_ordered", "w4_2procs",
        "w8_2procs"])
def test_ranks_in_processes(world, nprocs, n, dtype, variant, group, sync):
    import torch.multiprocessing as mp

    import dist_worker
    mp.spawn(dist_worker.run, args=(nprocs, dist_worker.free_port(), world, n, dtype, variant, 6, group, sync),
             nprocs=nprocs, join=True)


@pytest.mark.parametrize("world,n,dtype,variant", [
    (4, 4 * 32 * 300, "bf16", 0),
    (8, 8 * 32 * 512, "fp32", SENDER_EF),
    (2, 2 * 32 * 64, "bf16", OWNER_SUM),
])
def test_ranks_in_one_process(world, n, dtype, variant):
    """All ranks as handles of one process: the peers' buffers and events are
    used directly, with no CUDA IPC."""
    import dist_worker
    dist_worker.run(0, 1, 0, world, n, dtype, variant, 6, 32)


def test_connect_checks_the_blobs():
    """echo_dist_connect refuses blobs of another shape or in the wrong rank
    order, with nothing opened, and accepts the right ones afterwards."""
    import torch

    from bit_error_compensated_rank_b200 import echo
    torch.cuda.set_device(0)
    n = 2 * 32 * 64
    d0 = echo.DistEcho(2, 0, n)
    d1 = echo.DistEcho(2, 1, n)
    other = echo.DistEcho(2, 1, 2 * n)
    try:
        for blobs, words in [([d0.export(), other.export()], "expected rank 1"),
                             ([d1.export(), d0.export()], "expected rank 0")]:
            with pytest.raises(echo.EchoError) as ei:
                d0.connect(blobs)
            assert ei.value.code == echo.ECHO_ERR_INVALID and words in str(ei.value)
        blobs = [d0.export(), d1.export()]
        d0.connect(blobs)
        d1.connect(blobs)
        with pytest.raises(echo.EchoError):
            d0.connect(blobs)  # once per handle
        x = [torch.randn(n, device="cuda").to(torch.bfloat16) for _ in range(2)]
        out = [torch.empty_like(t) for t in x]
        echo.dist_allreduce([d0, d1], x, out, lambda: None)
        torch.cuda.synchronize()
        assert torch.equal(out[0].view(torch.int16), out[1].view(torch.int16))
    finally:
        torch.cuda.synchronize()
        for d in (d0, d1, other):
            d.close()
