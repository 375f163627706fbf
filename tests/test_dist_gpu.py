"""The all-reduce with one process per rank (echo_dist_*), several processes
on one GPU: each holds only its own partial and the state of the segment it
owns, the kernels store the wire straight into the other processes' blocks
(CUDA IPC), and every rank's result and owned state must equal the oracle's
bit for bit, call after call, for both phases, in place and out of place.

No kernel waits on another process: the stages are ordered by host barriers
(gloo), so the processes can share one GPU."""
import pytest

from oracle.oracle import FP16_SCALE, OWNER_SUM, SENDER_EF

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world,n,dtype,variant,group", [
    (2, 2 * 32 * 300, "bf16", 0, 32),
    (4, 4 * 32 * 129, "fp32", 0, 32),
    (3, 3 * 32 * 64, "bf16", OWNER_SUM | SENDER_EF, 32),
    (4, 4 * 128 * 40, "bf16", FP16_SCALE, 128),
    (2, 2 * 32 * 5000, "bf16", SENDER_EF, 16),
], ids=["w2", "w4_fp32", "w3_both", "w4_fp16_g128", "w2_ef_g16"])
def test_one_process_per_rank(world, n, dtype, variant, group):
    import torch.multiprocessing as mp

    import dist_worker
    mp.spawn(dist_worker.run, args=(world, dist_worker.free_port(), n, dtype, variant, 6, group),
             nprocs=world, join=True)
