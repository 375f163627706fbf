"""The debug build (libecho_debug.so) on the GPU: the parity suites run
against it with every index and copy range checked on the device and guard
bytes around every library buffer, and every call must leave the device
status word at 0; a guard byte changed from the host must be reported.

compute-sanitizer is not available on this GPU pool, so these checks stand in
for its memory checker: out-of-range accesses are skipped and recorded
(ECHO_STATUS_BOUNDS) instead of faulting, and a write past a buffer changes a
guard byte (ECHO_STATUS_CANARY)."""
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run_debug(args, timeout=1800):
    env = dict(os.environ, ECHO_LIB="debug")
    return subprocess.run([sys.executable] + args, cwd=ROOT, env=env, timeout=timeout,
                          capture_output=True, text=True)


def test_parity_suites_under_the_debug_build():
    res = _run_debug(["-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                      "tests/test_parity_gpu.py", "tests/test_variants_gpu.py",
                      "tests/test_groups_gpu.py", "tests/test_fp16_scale_gpu.py", "tests/test_dist_gpu.py",
                      "tests/test_fused_gpu.py",
                      "-k", "not one_gib and not largest and not error_growth and not timing"])
    assert res.returncode == 0, res.stdout[-4000:] + res.stderr[-2000:]


def test_guard_byte_change_is_reported():
    code = r"""
import numpy as np, torch
from bit_error_compensated_rank_b200 import echo
assert echo.echo_debug_build()
P, n = 4, 4 * 32 * 10
h = echo.Echo(P, n)
bufs = [torch.randn(n, device="cuda").to(torch.bfloat16) for _ in range(P)]
h.allreduce(bufs)
assert h.device_status(clear=True) == 0
h.debug_touch_guard()
h.allreduce(bufs)
st = h.device_status(clear=True)
assert st == echo.ECHO_STATUS_CANARY, st
h.close()
print("ok")
"""
    res = _run_debug(["-c", code], timeout=300)
    assert res.returncode == 0 and "ok" in res.stdout, res.stdout + res.stderr


def test_release_build_has_no_guards():
    import torch
    from bit_error_compensated_rank_b200 import echo
    if echo.echo_debug_build():
        pytest.skip("this process runs the debug build")
    h = echo.Echo(2, 2 * 32 * 4)
    try:
        with pytest.raises(echo.EchoError) as ei:
            h.debug_touch_guard()
        assert ei.value.code == echo.ECHO_ERR_UNSUPPORTED
        bufs = [torch.zeros(2 * 32 * 4, device="cuda", dtype=torch.bfloat16) for _ in range(2)]
        h.allreduce(bufs)
        assert h.device_status(clear=True) == 0
    finally:
        h.close()
