"""The benchmark's byte counts for the two ways a call can run (CPU only).

The one-kernel path (small calls) reads the P partials and the state once and
writes both wires, the state and the P outputs; the three pipelined kernels
also read the stage-1 wire and the requantised wire back and read the state
twice. bench.py reports each path against its own bytes, so these counts are
pinned here by hand to their per-element terms, and the difference between
the paths is checked to be exactly the reads the one kernel skips."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


@pytest.mark.parametrize("P", [2, 8, 16])
@pytest.mark.parametrize("b", [2, 4])
def test_fused_bytes_by_term(P, b):
    import bench
    n = P * 128 * 64
    wire = n // 2 + n // 32  # half a byte per code, one scale byte per group of 32
    reads = P * b * n + 8 * n  # partials, f and s
    writes = (P + 1) * wire + 8 * n + P * b * n  # both wires, f and s, the P outputs
    assert bench.fused_bytes(P, n, b) == reads + writes
    assert bench.fused_bytes(P, n, b, enable=False) == reads + writes - 16 * n
    # sender feedback: every rank's error read and written
    assert bench.fused_bytes(P, n, b, variant=2) == reads + writes + 8 * P * n
    # binary16 scales: two bytes per group
    assert bench.fused_bytes(P, n, b, variant=4) == reads + writes + (P + 1) * (n // 32)
    # groups of 128: one scale byte per 128 elements
    wire128 = n // 2 + n // 128
    assert bench.fused_bytes(P, n, b, group=128) == reads + (P + 1) * wire128 + 8 * n + P * b * n


def test_fused_bytes_against_the_three_kernels_on_one_gpu():
    """At P = 8 in bf16 the one kernel moves 52.78 B per element. The three
    kernels' single-GPU minimum is 65.56. The difference is the stage-1 wire
    read by kernel 2, the requantised wire read by kernel 3 and the state read
    again by kernel 2: 8 * 17/32 + 17/32 + 8 = 12.78 B."""
    import bench
    P, n = 8, 1 << 20
    assert bench.fused_bytes(P, n, 2) / n == pytest.approx(52.78125)
    single_gpu_min = 65.5625  # the benchmark line's single_gpu_min_bytes_per_elem at P = 8
    assert single_gpu_min - bench.fused_bytes(P, n, 2) / n == pytest.approx(P * 17 / 32 + 17 / 32 + 8)


def test_call_path_follows_the_limit():
    import bench

    class Handle:
        def __init__(self, limit):
            self.limit = limit

        def fused_limit(self):
            return self.limit

    assert bench.call_path(Handle(1 << 20), 1 << 20) == "one kernel"
    assert bench.call_path(Handle(1 << 20), (1 << 20) + 256) == "three kernels"
    assert bench.call_path(Handle(0), 4096) == "three kernels"
