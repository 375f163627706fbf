"""The sharded mode's host logic on CPU (no GPU): how the P ranks split over
the processes, the wire bytes that cross between GPUs, the argument checks,
and, with two gloo processes, the stage ordering of ``dist_allreduce``: no
process enqueues a stage of a call before every process has enqueued the
previous stage, and the host never waits for a stream."""
import json
import os
import socket
import subprocess
import sys
import time

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shard_ranks_split_evenly():
    import bench
    assert [bench.shard_ranks(8, 1, 0)] == [list(range(8))]
    assert [bench.shard_ranks(8, 2, r) for r in range(2)] == [[0, 1, 2, 3], [4, 5, 6, 7]]
    assert [bench.shard_ranks(8, 8, r) for r in range(8)] == [[r] for r in range(8)]
    with pytest.raises(ValueError):
        bench.shard_ranks(8, 3, 0)


@pytest.mark.parametrize("P,n_gpus", [(8, 1), (8, 2), (8, 4), (8, 8), (4, 4), (16, 8)])
def test_cross_gpu_link_bytes(P, n_gpus):
    """A GPU holding L = P/N ranks sends L (P - L) segments at stage 1 and
    L (P - L) requantised segments at stage 2, each W/P bytes for a message
    of W wire bytes; at one rank per GPU that is 2 (P-1)/P * W, the per-GPU
    share of the P-GPU link bytes 2 (P-1) W."""
    import bench
    n = P * 32 * 1024
    W = n // 2 + n // 32  # wire bytes of one message at group 32
    link = 2 * (P - 1) * W
    got = bench.cross_gpu_link_bytes(P, n_gpus, link)
    L = P // n_gpus
    # count segment by segment: rank r sends segment s to owner s, owner s
    # sends its total to rank r, whenever r and s sit on different GPUs
    seg = W // P
    count = sum(2 * seg for r in range(L) for s in range(P) if s // L != 0)
    assert got == count
    if n_gpus == P:
        assert got * P == link
    if n_gpus == 1:
        assert got == 0


@pytest.mark.parametrize("argv,env,msg", [
    (["--mode", "simulated", "--gpus", "2"], {"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"},
     "simulated mode runs one process"),
    (["--mode", "sharded", "--gpus", "3"], {"WORLD_SIZE": "3", "RANK": "1", "LOCAL_RANK": "1"},
     "does not split evenly"),
    (["--one-gpu", "--gpus", "2"], {"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"},
     "--one-gpu"),
    (["--mode", "replicas", "--host-ordered"], {}, "belong to the sharded mode"),
])
def test_bench_rejects_bad_mode_arguments(argv, env, msg):
    res = subprocess.run([sys.executable, "bench.py"] + argv, cwd=ROOT, capture_output=True, text=True,
                         env=dict(os.environ, **env), timeout=120)
    assert res.returncode == 2, res.stdout + res.stderr
    assert msg in res.stderr


class _FakeRank:
    """Stands in for a DistEcho handle: records when each stage is enqueued."""

    def __init__(self, rank, log, delay):
        self.rank, self.log, self.delay = rank, log, delay

    def stage(self, k, x, out, phase, stream):
        time.sleep(self.delay)
        self.log.append((time.monotonic(), self.rank, k))


class _NoSyncStream:
    def synchronize(self):
        raise AssertionError("the event-ordered form never waits for the stream")


def _ordering_worker(proc, nprocs, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    from bit_error_compensated_rank_b200 import echo

    dist.init_process_group("gloo", rank=proc, world_size=nprocs)
    log = []
    mine = bench.shard_ranks(8, nprocs, proc)
    ranks = [_FakeRank(r, log, 0.002 * (proc + 1)) for r in mine]
    for call in range(3):
        echo.dist_allreduce(ranks, [None] * len(ranks), [None] * len(ranks), dist.barrier,
                            stream=_NoSyncStream())
        log.append((time.monotonic(), -1, 10 + call))  # call returned
    with open(os.path.join(out_dir, f"p{proc}.json"), "w") as fh:
        json.dump(log, fh)
    dist.barrier()
    dist.destroy_process_group()


def test_stage_ordering_over_two_gloo_processes(tmp_path):
    pytest.importorskip("bit_error_compensated_rank_b200.echo")
    port = _free_port()
    mp.start_processes(_ordering_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    logs = [json.load(open(tmp_path / f"p{p}.json")) for p in range(2)]
    for log in logs:
        ends = [i for i, e in enumerate(log) if e[1] == -1]
        assert len(ends) == 3
    # split every process's log into calls, then check the barrier order
    calls = []
    for log in logs:
        per_call, cur = [], []
        for t, r, k in log:
            if r == -1:
                per_call.append(cur)
                cur = []
            else:
                cur.append((t, r, k))
        calls.append(per_call)
    for c in range(3):
        for k in (2, 3):
            first_k = min(t for p in range(2) for t, r, kk in calls[p][c] if kk == k)
            last_prev = max(t for p in range(2) for t, r, kk in calls[p][c] if kk == k - 1)
            assert first_k >= last_prev, (c, k)
        for p in range(2):
            stages = [kk for _, _, kk in calls[p][c]]
            assert stages == [1] * 4 + [2] * 4 + [3] * 4  # every held rank, stage by stage
