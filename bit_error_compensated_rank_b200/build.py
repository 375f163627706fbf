"""Build ``libecho.so`` in-tree with nvcc for sm_100a.

    python -m bit_error_compensated_rank_b200.build [--verbose] [--debug | --all]

``--debug`` builds ``libecho_debug.so`` instead: the same sources with
``ECHO_DEBUG=1`` (device-side bounds checks on every computed index and copy
range, guard bytes around every library buffer, both reported through the
device status word). ``--all`` builds both.

Each ``csrc/*.cu`` compiles to an object under ``_build/`` (in parallel), then
nvcc links them into ``bit_error_compensated_rank_b200/lib/libecho.so`` with the
CUDA runtime linked statically, so loading the library needs no CUDA install
beyond the driver. Floating-point flags keep IEEE binary32 semantics exactly
(no flush to zero, no fused multiply-add contraction, IEEE division and square
root): the kernels must reproduce the oracle's arithmetic bit for bit.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_DIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIB_DIR, "libecho.so")
OBJ_DIR = os.path.join(ROOT, "_build", "echo")
LIB_DEBUG = os.path.join(LIB_DIR, "libecho_debug.so")
OBJ_DIR_DEBUG = os.path.join(ROOT, "_build", "echo_debug")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + [
    "-O3", "-lineinfo", "-std=c++17",
    "-ftz=false", "-prec-div=true", "-prec-sqrt=true", "-fmad=false",
    "-Xcompiler", "-fPIC,-fvisibility=hidden,-Wall",
    "-I", INCLUDE, "-I", CSRC,
]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found: the CUDA library cannot be built")
    return path


def sources() -> list[str]:
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def headers() -> list[str]:
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    return hs + [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]


def _stale(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src: str, obj: str, verbose: bool, debug: bool = False) -> str:
    cmd = [nvcc()] + NVCC_FLAGS + (["-DECHO_DEBUG=1"] if debug else []) + ["-c", src, "-o", obj]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n{res.stdout}\n{res.stderr}")
    return res.stdout + res.stderr


def build(verbose: bool = False, force: bool = False, debug: bool = False) -> str:
    """Compile what changed and link ``libecho.so`` (``libecho_debug.so``
    with debug); return its path."""
    obj_dir = OBJ_DIR_DEBUG if debug else OBJ_DIR
    lib = LIB_DEBUG if debug else LIB
    os.makedirs(obj_dir, exist_ok=True)
    os.makedirs(LIB_DIR, exist_ok=True)
    hdrs = headers()
    jobs = []
    objs = []
    for src in sources():
        obj = os.path.join(obj_dir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if force or verbose or _stale(obj, [src] + hdrs):
            jobs.append((src, obj))
    logs = []
    if jobs:
        with cf.ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 4)) as ex:
            futs = [ex.submit(_compile, s, o, verbose, debug) for s, o in jobs]
            for f in futs:
                logs.append(f.result())
    if jobs or _stale(lib, objs):
        cmd = [nvcc()] + ARCH + ["-shared", "-cudart", "static", "-o", lib] + objs + ["-ldl"]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError(f"link failed:\n{res.stdout}\n{res.stderr}")
    if verbose:
        sys.stdout.write("".join(logs))
    return lib


def build_all(verbose: bool = False, force: bool = False) -> list[str]:
    """The release library and the debug library."""
    return [build(verbose, force, debug=False), build(verbose, force, debug=True)]


if __name__ == "__main__":
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--verbose", action="store_true", help="print ptxas resource usage")
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--debug", action="store_true", help="build libecho_debug.so instead")
    ap.add_argument("--all", action="store_true", help="build both libraries")
    args = ap.parse_args()
    if args.all:
        print("\n".join(build_all(verbose=args.verbose, force=args.force)))
    else:
        print(build(verbose=args.verbose, force=args.force, debug=args.debug))
