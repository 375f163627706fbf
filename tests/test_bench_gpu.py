"""The benchmark's own code paths on the GPU, at small sizes: the simulated
line, the sharded mode (ranks as handles of one process, and two processes
sharing one GPU under torchrun), and a per-workload line. Each must exit 0
and print one JSON line whose fields hold together; the numbers themselves
are not checked here."""
import json
import os
import socket
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, timeout=600):
    res = subprocess.run([sys.executable] + args, cwd=ROOT, capture_output=True, text=True, timeout=timeout)
    assert res.returncode == 0, res.stdout[-3000:] + res.stderr[-3000:]
    return json.loads(res.stdout.strip().splitlines()[-1])


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_simulated_line():
    n = 8 * 32 * 4096
    line = _run(["bench.py", "--elems", str(n), "--steps", "5", "--warmup", "3", "--no-cpu-baseline",
                 "--e2e-steps", "1"])
    assert line["config"]["mode"] == "simulated" and line["n_gpus"] == 1
    assert line["config"]["n_per_rank"] == n
    assert line["value"] > 0 and line["roofline"]["bound"] == "hbm"
    assert 0 < line["single_gpu_min_frac"] < line["hbm_roofline_frac"]
    assert line["e2e"]["h2d_bytes_per_step"] == 8 * n * 2 and line["e2e"]["d2h_bytes_per_step"] == n * 2
    assert line["gpu_launches"] == 3 * 5


def test_sharded_line_in_one_process():
    n = 8 * 32 * 4096
    line = _run(["bench.py", "--mode", "sharded", "--elems", str(n), "--steps", "5", "--warmup", "3",
                 "--e2e-steps", "1"])
    assert line["config"]["mode"] == "sharded" and line["scaling"] == "strong"
    assert line["n_gpus"] == 1 and line["link_bytes_per_gpu_per_call"] == 0
    assert len(line["stage_ms"]) == 3 and all(t > 0 for t in line["stage_ms"])
    assert line["gpu_launches"] == 3 * 8 * 5
    assert line["e2e"]["h2d_bytes_per_step"] == 8 * n * 2


def test_sharded_line_two_processes_one_gpu():
    n = 4 * 32 * 2048
    cmd = ["-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2", "--master-addr",
           "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--gpus", "1", "--one-gpu",
           "--mode", "sharded", "--ranks", "4", "--elems", str(n), "--steps", "5", "--warmup", "3",
           "--no-e2e"]
    line = _run(cmd)
    assert line["config"]["mode"] == "sharded" and line["config"]["P"] == 4
    assert "2 process(es) on 1 GPU(s)" in line["config"]["parallelism"]
    assert line["gpu_launches"] == 3 * 2 * 5  # this process's two ranks


def test_workload_line():
    line = _run(["bench.py", "--config", "1", "--warmup", "3"])
    assert line["config_line"] == 1 and line["regime"] == "launch-bound"
    assert line["us_per_call_graph"] > 0 and line["us_per_call_eager"] > 0
