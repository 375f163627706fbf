"""The C ABI without a GPU: the library loads, exports every entry point the
header declares, and rejects bad arguments before touching CUDA."""
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "echo.h")


@pytest.fixture(scope="module")
def echo():
    from bit_error_compensated_rank_b200 import build
    build.build()
    from bit_error_compensated_rank_b200 import echo as mod
    return mod


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"ECHO_API\s+[\w\s\*]*?\b(echo_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for required in ("echo_create", "echo_allreduce", "echo_reset", "echo_destroy",
                     "echo_last_error", "echo_set_params", "echo_get_state", "echo_set_state",
                     "echo_get_wire", "echo_stats"):
        assert required in names


def test_debug_library_exports_the_same_symbols(echo):
    from bit_error_compensated_rank_b200 import build
    path = build.build(debug=True)
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True,
                         text=True, check=True).stdout
    assert set(re.findall(r"\bT (echo_\w+)", out)) == set(declared_symbols())


def test_build_flavour_is_reported(echo):
    assert echo.echo_debug_build() is False
    code = ("from bit_error_compensated_rank_b200 import echo; "
            "assert echo.LIB_PATH.endswith('libecho_debug.so'); assert echo.echo_debug_build()")
    env = dict(os.environ, ECHO_LIB="debug")
    subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, check=True)


def test_library_exports_every_declared_symbol(echo):
    out = subprocess.run(["nm", "-D", "--defined-only", echo.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (echo_\w+)", out))
    declared = set(declared_symbols())
    assert declared <= exported, declared - exported
    assert exported <= declared, exported - declared  # nothing undeclared leaks
    assert set(echo.EXPORTED) == declared


def test_model_bytes_per_element(echo):
    # P*b + 8 + P*w | P*w + 16 + w | P*w + P*b per element, w = 17/32
    P, n = 8, 1 << 29
    mb = echo.echo_model_bytes(P, n, echo.ECHO_BF16, True)
    w = 17 / 32
    assert mb["k1"] == round((P * 2 + 8 + P * w) * n)
    assert mb["k2"] == round((P * w + 16 + w) * n)
    assert mb["k3"] == round((P * w + P * 2) * n)
    assert mb["link"] == round(2 * (P - 1) * w * n)
    assert abs(mb["total"] / n - 69.28125) < 1e-12
    off = echo.echo_model_bytes(P, n, echo.ECHO_BF16, False)
    assert mb["total"] - off["total"] == 24 * n
    f32 = echo.echo_model_bytes(8, 65536, echo.ECHO_FP32, True)
    assert abs(f32["total"] / 65536 - (2 * 8 * 4 + 25 * w + 24)) < 1e-12


def test_link_bytes_are_17_64_of_a_16_bit_exchange(echo):
    """The pages' "almost four times" less volume [rit.work "Echo 4-bit GPU
    communication", first section]: the counted link bytes of one call are
    17/64 of those of the same reduce-scatter + all-gather in 16 bits."""
    from fractions import Fraction
    for P, n in [(2, 4096), (4, 2048 * 4096), (8, 1 << 29), (16, 16 * 32 * 1000)]:
        mb = echo.echo_model_bytes(P, n, echo.ECHO_BF16, True)
        assert Fraction(mb["link"], 2 * (P - 1) * n * 2) == Fraction(17, 64)


@pytest.mark.parametrize("fp16", [False, True])
@pytest.mark.parametrize("group", [16, 32, 64, 128])
def test_model_bytes_group_sizes(echo, group, fp16):
    # the wire costs 1/2 + 1/group bytes per element (2/group with binary16
    # scales), the rest is unchanged
    P, n = 8, 1 << 29
    mb = echo.echo_model_bytes_ex(P, n, group, echo.ECHO_BF16, True,
                                  echo.ECHO_VARIANT_FP16_SCALE if fp16 else 0)
    w = 0.5 + (2 if fp16 else 1) / group
    assert mb["k1"] == round((P * 2 + 8 + P * w) * n)
    assert mb["k2"] == round((P * w + 16 + w) * n)
    assert mb["k3"] == round((P * w + P * 2) * n)
    assert mb["link"] == round(2 * (P - 1) * w * n)


@pytest.mark.parametrize("P,n,group,dtype,status", [
    (1, 64, 32, 0, -1), (17, 17 * 32, 32, 0, -1), (2, 0, 32, 0, -1), (2, 96, 32, 0, -1),
    (4, 4 * 32 * 3 + 32, 32, 0, -1), (2, 64, 32, 7, -1), (2, 192, 48, 0, -2),
    (2, 512, 256, 0, -2), (2, 64, 8, 0, -2), (4, 4 * 64 * 3 + 64, 64, 0, -1),
    (5, 5 * 16, 16, 0, -2),
    (2, 1 << 35, 32, 0, -2), (2, 64, 0, 0, -1),
])
def test_create_rejects_bad_shapes(echo, P, n, group, dtype, status):
    with pytest.raises(echo.EchoError) as ei:
        echo.echo_create(P, n, group, dtype)
    assert ei.value.code == status
    assert echo.echo_last_status() == status
    assert echo.echo_last_error()


@pytest.mark.parametrize("world,rank,n,group,dtype,status", [
    (1, 0, 64, 32, 0, -1), (17, 0, 17 * 32, 32, 0, -1), (2, 2, 64, 32, 0, -1), (2, -1, 64, 32, 0, -1),
    (2, 0, 96, 32, 0, -1), (2, 0, 2 * 48, 48, 0, -2), (2, 0, 64, 32, 9, -1), (3, 0, 3 * 16, 16, 0, -1),
])
def test_dist_create_rejects_bad_shapes(echo, world, rank, n, group, dtype, status):
    assert not echo._lib.echo_dist_create(world, rank, n, group, dtype)
    assert echo.echo_last_status() == status
    assert echo.echo_last_error()


def test_null_and_unknown_handles(echo):
    for fn, args in [(echo._lib.echo_allreduce, (None, None, 0, None)),
                     (echo._lib.echo_reset, (None, 1)),
                     (echo._lib.echo_set_params, (None, 0.5, 0.875, 0.5, 1)),
                     (echo._lib.echo_stats, (None, None, None, None)),
                     (echo._lib.echo_set_timing, (None, 1)),
                     (echo._lib.echo_set_fused_limit, (None, 0)),
                     (echo._lib.echo_get_fused_limit, (None, None))]:
        assert fn(*args) == echo.ECHO_ERR_INVALID
        assert "NULL" in echo.echo_last_error()
    bogus = 0x1000
    assert echo._lib.echo_reset(bogus, 1) == echo.ECHO_ERR_INVALID
    assert "unknown or destroyed" in echo.echo_last_error()
    assert echo._lib.echo_destroy(None) == echo.ECHO_OK


def test_injected_allocation_failure():
    code = (
        "import os; os.environ['ECHO_FAULT'] = 'alloc'\n"
        "from bit_error_compensated_rank_b200 import echo as e\n"
        "try:\n"
        "    e.echo_create(2, 64)\n"
        "    raise SystemExit('no error')\n"
        "except e.EchoError as err:\n"
        "    assert err.code == e.ECHO_ERR_OOM, err\n"
        "    assert 'injected' in str(err)\n"
    )
    res = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr + res.stdout


def test_binding_fails_loudly_without_library(tmp_path):
    """The binding has no fallback: with the library missing, import fails."""
    code = (
        "import sys, os, importlib.util\n"
        "spec = importlib.util.spec_from_file_location('echo_copy', sys.argv[1])\n"
        "mod = importlib.util.module_from_spec(spec)\n"
        "try:\n"
        "    spec.loader.exec_module(mod)\n"
        "except ImportError as e:\n"
        "    assert 'no fallback' in str(e)\n"
        "    sys.exit(0)\n"
        "sys.exit(1)\n"
    )
    copy = tmp_path / "echo.py"
    copy.write_text(open(os.path.join(ROOT, "bit_error_compensated_rank_b200", "echo.py")).read())
    res = subprocess.run([sys.executable, "-c", code, str(copy)], capture_output=True, text=True)
    assert res.returncode == 0, res.stderr


@pytest.mark.parametrize("P,n,dtype,params,status,words", [
    (1, 64, 0, (0.5, 0.875, 0.5, 1), -1, "outside"),
    (17, 17 * 32, 0, (0.5, 0.875, 0.5, 1), -1, "outside"),
    (2, 64, 5, (0.5, 0.875, 0.5, 1), -1, "dtype"),
    (2, 0, 0, (0.5, 0.875, 0.5, 1), -1, "multiple"),
    (4, 4 * 32 * 3 + 32, 0, (0.5, 0.875, 0.5, 1), -1, "multiple"),
    (2, 64, 0, (1.0, 0.875, 0.5, 1), -1, "parameters"),
    (2, 64, 0, (0.5, -0.1, 0.5, 1), -1, "parameters"),
    (2, 64, 0, (0.5, 0.875, 1.5, 1), -1, "parameters"),
    (2, 64, 0, (0.5, 0.875, 0.5, 2), -1, "parameters"),
    # larger than the fixed scratch array
    (8, 8 * 32 * 65536, 0, (0.5, 0.875, 0.5, 1), -2, "static scratch"),
    # past 2^34, including a size whose scratch arithmetic would wrap around
    # 64 bits: rejected before any of it is computed
    (16, (1 << 34) + 512, 0, (0.5, 0.875, 0.5, 1), -2, "maximum"),
    (16, (1 << 64) - 512, 1, (0.5, 0.875, 0.5, 1), -2, "maximum"),
])
def test_static_rejects_bad_arguments_before_cuda(echo, P, n, dtype, params, status, words):
    """echo_allreduce_static checks its shape and parameters on the host,
    before any CUDA call, so these run without a GPU; pointer checks need one
    and run in the GPU suite."""
    bf, bs, lam, en = params
    ptrs = echo._ptr_array([0] * max(P, 1))
    rc = echo._lib.echo_allreduce_static(P, n, dtype, ptrs, None, None, bf, bs, lam, en, None)
    assert rc == status, echo.echo_last_error()
    assert echo.echo_last_status() == status
    assert words in echo.echo_last_error()


def test_static_status_needs_an_output(echo):
    assert echo._lib.echo_static_status(None, 0) == echo.ECHO_ERR_INVALID
    assert "NULL" in echo.echo_last_error()


C_CLIENT = r"""
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "echo.h"

/* A plain C99 client of the boundary: only calls that need no GPU. */
int main(void)
{
    uint64_t out[4];
    const size_t n = (size_t)8 * 32 * 1024;
    echo_handle *h;
    uint8_t blob[ECHO_DIST_HANDLE_BYTES];

    if (echo_model_bytes(8, n, ECHO_BF16, 1, out) != ECHO_OK)
        return 1;
    /* P*b + 8 + P*w, P*w + 16 + w, P*w + P*b bytes per element (w = 17/32) */
    if (out[0] != n * 16 + n * 8 + 8 * (n / 2 + n / 32))
        return 2;
    if (out[1] != 8 * (n / 2 + n / 32) + n * 16 + (n / 2 + n / 32))
        return 3;
    if (out[2] != 8 * (n / 2 + n / 32) + n * 16)
        return 4;
    if (out[3] != (uint64_t)2 * 7 * (n / 2 + n / 32))
        return 5;
    h = echo_create(1, n, 32, ECHO_BF16); /* P = 1 is refused before CUDA is touched */
    if (h != NULL || echo_last_status() != ECHO_ERR_INVALID || strlen(echo_last_error()) == 0)
        return 6;
    if (echo_allreduce(NULL, NULL, ECHO_FWD, NULL) != ECHO_ERR_INVALID)
        return 7;
    if (echo_set_fused_limit(NULL, 0) != ECHO_ERR_INVALID)
        return 8;
    if (echo_destroy(NULL) != ECHO_OK)
        return 9;
    if (echo_dist_export(NULL, blob) != ECHO_ERR_INVALID)
        return 10;
    printf("ok\n");
    return 0;
}
"""


def test_header_compiles_as_c99_and_links(echo, tmp_path):
    """The boundary as a C user sees it: the header compiles as strict C99
    (no C++), the program links against libecho.so, and the calls that need no
    GPU give the documented results."""
    src = tmp_path / "client.c"
    exe = tmp_path / "client"
    src.write_text(C_CLIENT)
    lib_dir = os.path.dirname(echo.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
                    os.path.join(ROOT, "include"), str(src), "-o", str(exe), "-L", lib_dir, "-lecho",
                    "-Wl,-rpath," + lib_dir], check=True, capture_output=True, text=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True)
    assert res.returncode == 0 and res.stdout.strip() == "ok", (res.returncode, res.stdout, res.stderr)
