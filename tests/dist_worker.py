"""Ranks of the one-rank-per-handle tests (tests/test_dist_gpu.py): run as a
spawned process (or called directly for a single process), it holds one or
more consecutive ranks, all-reduces their partials with the other ranks
through the echo_dist_* entry points and checks every held rank's result and
owned state against the oracle, computed here from the same seeded inputs."""
from __future__ import annotations

import datetime

import numpy as np


def run(proc: int, nprocs: int, port: int, world: int, n: int, dtype: str, variant: int, calls: int,
        group: int, sync: bool = False):
    import torch
    import torch.distributed as dist

    from bit_error_compensated_rank_b200 import echo
    from bit_error_compensated_rank_b200 import workloads as wl
    from gpu_harness import assert_same_bits
    from oracle.oracle import Oracle, Params

    if nprocs > 1:
        dist.init_process_group("gloo", rank=proc, world_size=nprocs, init_method=f"tcp://127.0.0.1:{port}",
                                timeout=datetime.timedelta(seconds=120))
        barrier = dist.barrier
    else:
        def barrier():
            return None
    try:
        torch.cuda.set_device(0)
        per = world // nprocs
        mine = list(range(proc * per, (proc + 1) * per))
        code = echo.ECHO_BF16 if dtype == "bf16" else echo.ECHO_FP32
        ds = [echo.DistEcho(world, r, n, code, group) for r in mine]
        for d in ds:
            if variant:
                d.set_variant(variant)
        blobs = [d.export() for d in ds]
        if nprocs > 1:
            gathered = [None] * nprocs
            dist.all_gather_object(gathered, blobs)
            blobs = [b for part in gathered for b in part]
        for d in ds:
            d.connect(blobs)
        orc = Oracle()
        f = {ph: np.zeros(n, np.float32) for ph in (0, 1)}
        s = {ph: np.zeros(n, np.float32) for ph in (0, 1)}
        eps = {ph: np.zeros((world, n), np.float32) for ph in (0, 1)}
        for k in range(calls):
            phase = (k // 2) & 1
            xs = wl.outlier_gaussian(world, n, seed=60 + world, call=k, dtype=dtype)  # every rank's partial
            xt, outs = [], []
            for r in mine:
                part = np.ascontiguousarray(xs[r])
                if dtype == "bf16":
                    x = torch.from_numpy(part.view(np.int16)).cuda().view(torch.bfloat16)
                else:
                    x = torch.from_numpy(part).cuda()
                xt.append(x)
                outs.append(torch.empty_like(x) if k % 3 else x)  # in place every third call
            echo.dist_allreduce(ds, xt, outs, barrier, phase=phase, sync=sync)
            ref = orc.allreduce(xs, f[phase], s[phase], Params(), G=group, variant=variant, eps=eps[phase])
            for r, d, out in zip(mine, ds, outs):
                got = out.view(torch.int16).cpu().numpy().view(np.uint16) if dtype == "bf16" \
                    else out.cpu().numpy()
                assert_same_bits(got, ref["out"], f"rank {r} call {k} output")
                seg = slice(r * (n // world), (r + 1) * (n // world))
                for ph in (0, 1):
                    gf, gs = d.get_state(ph)
                    assert_same_bits(gf, f[ph][seg], f"rank {r} call {k} fast estimate phase {ph}")
                    assert_same_bits(gs, s[ph][seg], f"rank {r} call {k} slow estimate phase {ph}")
                assert d.device_status(clear=True) == 0
        torch.cuda.synchronize()
        barrier()
        for d in ds:
            d.close()
    finally:
        if nprocs > 1:
            dist.barrier()
            dist.destroy_process_group()


def free_port() -> int:
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as sock:
        sock.bind(("127.0.0.1", 0))
        return sock.getsockname()[1]
