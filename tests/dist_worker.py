"""One rank of the one-process-per-rank tests (tests/test_dist_gpu.py): run
as a spawned process, it all-reduces its own partial with the others through
the echo_dist_* entry points and checks its result and its owned state
against the oracle, computed here from the same seeded inputs."""
from __future__ import annotations

import datetime

import numpy as np


def run(rank: int, world: int, port: int, n: int, dtype: str, variant: int, calls: int, group: int):
    import torch
    import torch.distributed as dist

    from bit_error_compensated_rank_b200 import echo
    from bit_error_compensated_rank_b200 import workloads as wl
    from gpu_harness import assert_same_bits
    from oracle.oracle import Oracle, Params

    dist.init_process_group("gloo", rank=rank, world_size=world, init_method=f"tcp://127.0.0.1:{port}",
                            timeout=datetime.timedelta(seconds=120))
    try:
        torch.cuda.set_device(0)
        d = echo.DistEcho(world, rank, n, echo.ECHO_BF16 if dtype == "bf16" else echo.ECHO_FP32, group)
        if variant:
            d.set_variant(variant)
        handles = [None] * world
        dist.all_gather_object(handles, d.export())
        d.connect(handles)
        orc = Oracle()
        f = {ph: np.zeros(n, np.float32) for ph in (0, 1)}
        s = {ph: np.zeros(n, np.float32) for ph in (0, 1)}
        eps = {ph: np.zeros((world, n), np.float32) for ph in (0, 1)}
        seg = slice(rank * (n // world), (rank + 1) * (n // world))
        for k in range(calls):
            phase = (k // 2) & 1
            xs = wl.outlier_gaussian(world, n, seed=60 + world, call=k, dtype=dtype)  # every rank's partial
            mine = np.ascontiguousarray(xs[rank])
            if dtype == "bf16":
                x = torch.from_numpy(mine.view(np.int16)).cuda().view(torch.bfloat16)
            else:
                x = torch.from_numpy(mine).cuda()
            out = torch.empty_like(x) if k % 3 else x  # in place every third call
            d.allreduce(x, out, dist.barrier, phase=phase)
            ref = orc.allreduce(xs, f[phase], s[phase], Params(), G=group, variant=variant, eps=eps[phase])
            got = out.view(torch.int16).cpu().numpy().view(np.uint16) if dtype == "bf16" else out.cpu().numpy()
            assert_same_bits(got, ref["out"], f"rank {rank} call {k} output")
            for ph in (0, 1):
                gf, gs = d.get_state(ph)
                assert_same_bits(gf, f[ph][seg], f"rank {rank} call {k} fast estimate phase {ph}")
                assert_same_bits(gs, s[ph][seg], f"rank {rank} call {k} slow estimate phase {ph}")
            assert d.device_status(clear=True) == 0
        dist.barrier()
        d.close()
    finally:
        dist.barrier()
        dist.destroy_process_group()


def free_port() -> int:
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as sock:
        sock.bind(("127.0.0.1", 0))
        return sock.getsockname()[1]

