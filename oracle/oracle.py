"""ctypes wrapper around the CPU oracle (``libecho_oracle.so``).

TEST INFRASTRUCTURE. Only the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this module. The CUDA library neither
imports nor links anything here; the two share no code. The method and the
readings the oracle fixes are described in ``echo_oracle.h``.

Arrays are numpy: bf16 values travel as ``uint16`` bit patterns, binary32 as
``float32``. Each call is single-threaded.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_NAME = "libecho_oracle.so"

BF16 = 0
FP32 = 1
OWNER_SUM = 1   # variant: the owner adds the correction to its sum
SENDER_EF = 2   # variant: every rank feeds back its own rounding-#1 error
FP16_SCALE = 4  # variant: binary16 scales (rounded up) instead of powers of two

_u8p = ctypes.POINTER(ctypes.c_uint8)
_i8p = ctypes.POINTER(ctypes.c_int8)
_f32p = ctypes.POINTER(ctypes.c_float)
_i32p = ctypes.POINTER(ctypes.c_int32)
_u16p = ctypes.POINTER(ctypes.c_uint16)


def build(src_dir: str = HERE) -> str:
    """Compile the oracle with its Makefile (no-op when up to date)."""
    subprocess.run(["make", "-s", "-C", src_dir], check=True)
    return os.path.join(src_dir, LIB_NAME)


def _ptr(a, ctype):
    if a is None:
        return None
    return a.ctypes.data_as(ctype)


@dataclass
class Params:
    """Compensator settings; the defaults are the fixed readings."""

    lam: float = 0.5
    beta_fast: float = 0.5
    beta_slow: float = 0.875
    enable: bool = True


class Oracle:
    """Handle on one build of the oracle library (a path may point at a
    deliberately altered copy: the mutation tests do that)."""

    def __init__(self, lib_path: str | None = None):
        if lib_path is None:
            lib_path = build()
        self.path = lib_path
        lib = ctypes.CDLL(lib_path)
        lib.echo_oracle_quantize_group.argtypes = [_f32p, ctypes.c_int, _i8p]
        lib.echo_oracle_quantize_group.restype = ctypes.c_int
        lib.echo_oracle_dequant.argtypes = [ctypes.c_int, ctypes.c_int]
        lib.echo_oracle_dequant.restype = ctypes.c_float
        lib.echo_oracle_pack.argtypes = [_i8p, ctypes.c_size_t, _u8p]
        lib.echo_oracle_pack.restype = None
        lib.echo_oracle_unpack.argtypes = [_u8p, ctypes.c_size_t, _i8p]
        lib.echo_oracle_unpack.restype = None
        lib.echo_oracle_quantize_group_f16.argtypes = [_f32p, ctypes.c_int, _i8p, _u16p]
        lib.echo_oracle_quantize_group_f16.restype = ctypes.c_int
        lib.echo_oracle_dequant_f16.argtypes = [ctypes.c_int, ctypes.c_uint16]
        lib.echo_oracle_dequant_f16.restype = ctypes.c_float
        lib.echo_oracle_half_value.argtypes = [ctypes.c_uint16]
        lib.echo_oracle_half_value.restype = ctypes.c_double
        lib.echo_oracle_round_bf16.argtypes = [ctypes.c_float]
        lib.echo_oracle_round_bf16.restype = ctypes.c_float
        common = [ctypes.c_void_p, ctypes.c_void_p, _f32p, _f32p,
                  ctypes.c_float, ctypes.c_float, ctypes.c_float, ctypes.c_int,
                  _u8p, _u8p, _u8p, _u8p, _f32p, _f32p]
        lib.echo_oracle_allreduce_groups.argtypes = (
            [ctypes.c_int, ctypes.c_int, ctypes.c_size_t, _i32p, ctypes.c_int] + common)
        lib.echo_oracle_allreduce_groups.restype = ctypes.c_int
        lib.echo_oracle_allreduce.argtypes = (
            [ctypes.c_int, ctypes.c_size_t, ctypes.c_int, ctypes.c_int] + common)
        lib.echo_oracle_allreduce.restype = ctypes.c_int
        common_ex = [ctypes.c_void_p, ctypes.c_void_p, _f32p, _f32p, _f32p,
                     ctypes.c_float, ctypes.c_float, ctypes.c_float, ctypes.c_int, ctypes.c_int,
                     _u8p, _u8p, _u8p, _u8p, _f32p, _f32p]
        lib.echo_oracle_allreduce_groups_ex.argtypes = (
            [ctypes.c_int, ctypes.c_int, ctypes.c_size_t, _i32p, ctypes.c_int] + common_ex)
        lib.echo_oracle_allreduce_groups_ex.restype = ctypes.c_int
        lib.echo_oracle_allreduce_ex.argtypes = (
            [ctypes.c_int, ctypes.c_size_t, ctypes.c_int, ctypes.c_int] + common_ex)
        lib.echo_oracle_allreduce_ex.restype = ctypes.c_int
        self.lib = lib

    # ---- codec -----------------------------------------------------------
    def quantize_group(self, v) -> tuple[int, np.ndarray]:
        v = np.ascontiguousarray(v, dtype=np.float32)
        q = np.zeros(v.shape[0], dtype=np.int8)
        b = self.lib.echo_oracle_quantize_group(_ptr(v, _f32p), v.shape[0], _ptr(q, _i8p))
        if b < 0:
            raise ValueError(f"oracle quantize_group failed ({b})")
        return b, q

    def dequant(self, q: int, b: int) -> float:
        return float(np.float32(self.lib.echo_oracle_dequant(int(q), int(b))))

    def quantize_group_f16(self, v) -> tuple[int, np.ndarray]:
        """Binary16 scale pattern and codes of one group (variant FP16_SCALE)."""
        v = np.ascontiguousarray(v, dtype=np.float32)
        q = np.zeros(v.shape[0], dtype=np.int8)
        h = ctypes.c_uint16(0)
        rc = self.lib.echo_oracle_quantize_group_f16(_ptr(v, _f32p), v.shape[0], _ptr(q, _i8p),
                                                     ctypes.byref(h))
        if rc < 0:
            raise ValueError(f"oracle quantize_group_f16 failed ({rc})")
        return int(h.value), q

    def dequant_f16(self, q: int, h: int) -> float:
        return float(np.float32(self.lib.echo_oracle_dequant_f16(int(q), int(h))))

    def half_value(self, h: int) -> float:
        return float(self.lib.echo_oracle_half_value(int(h)))

    def round_bf16(self, v: float) -> float:
        return float(np.float32(self.lib.echo_oracle_round_bf16(float(np.float32(v)))))

    def pack(self, q) -> np.ndarray:
        q = np.ascontiguousarray(q, dtype=np.int8)
        out = np.zeros(q.shape[0] // 2, dtype=np.uint8)
        self.lib.echo_oracle_pack(_ptr(q, _i8p), q.shape[0], _ptr(out, _u8p))
        return out

    def unpack(self, packed) -> np.ndarray:
        packed = np.ascontiguousarray(packed, dtype=np.uint8)
        q = np.zeros(packed.shape[0] * 2, dtype=np.int8)
        self.lib.echo_oracle_unpack(_ptr(packed, _u8p), q.shape[0], _ptr(q, _i8p))
        return q

    # ---- one all-reduce call ---------------------------------------------
    def allreduce(self, x, f=None, s=None, params: Params = Params(), G: int = 32,
                  owner=None, want_wire: bool = True, want_diag: bool = False,
                  variant: int = 0, eps=None) -> dict:
        """One call on rank partials ``x`` of shape (P, m).

        ``x`` is uint16 (bf16 bit patterns) or float32. ``f`` and ``s`` (float32,
        length m) are updated in place when compensation is on. ``owner`` (one
        rank per group) overrides the contiguous segment layout; it lets a
        caller run any subset of groups of a larger problem.
        ``variant`` is a bit set of OWNER_SUM, SENDER_EF and FP16_SCALE; with
        SENDER_EF, ``eps`` (float32, shape (P, m)) is every rank's rounding-#1
        error state, updated in place; with FP16_SCALE the scale arrays hold
        binary16 bit patterns (uint16) instead of scale bytes.
        Returns a dict with ``out`` and, if requested, the wire and diagnostics.
        """
        x = np.ascontiguousarray(x)
        if x.dtype == np.uint16:
            dtype = BF16
        elif x.dtype == np.float32:
            dtype = FP32
        else:
            raise TypeError("x must be uint16 (bf16 bits) or float32")
        P, m = x.shape
        if m % G:
            raise ValueError("m must be a multiple of G")
        ngroups = m // G
        if params.enable:
            if f is None or s is None:
                raise ValueError("compensation on needs f and s")
            for a in (f, s):
                if a.dtype != np.float32 or a.shape != (m,) or not a.flags.c_contiguous:
                    raise ValueError("f and s must be contiguous float32 of length m")
        if variant & SENDER_EF:
            if eps is None or eps.dtype != np.float32 or eps.shape != (P, m) or \
                    not eps.flags.c_contiguous:
                raise ValueError("SENDER_EF needs eps: contiguous float32 of shape (P, m)")
        out = np.zeros(m, dtype=x.dtype)
        res = {"out": out}
        if want_wire:
            res["codes1"] = np.zeros((P, m // 2), dtype=np.uint8)
            sdt = np.uint16 if variant & FP16_SCALE else np.uint8
            res["scales1"] = np.zeros((P, ngroups), dtype=sdt)
            res["qcodes"] = np.zeros(m // 2, dtype=np.uint8)
            res["qscales"] = np.zeros(ngroups, dtype=sdt)
        if want_diag:
            res["c"] = np.zeros(m, dtype=np.float32)
            res["err"] = np.zeros(m, dtype=np.float32)
        args = [x.ctypes.data, out.ctypes.data, _ptr(f, _f32p), _ptr(s, _f32p),
                _ptr(eps if variant & SENDER_EF else None, _f32p),
                params.lam, params.beta_fast, params.beta_slow, int(bool(params.enable)),
                int(variant),
                _ptr(res.get("codes1"), _u8p), _ptr(res.get("scales1"), _u8p),
                _ptr(res.get("qcodes"), _u8p), _ptr(res.get("qscales"), _u8p),
                _ptr(res.get("c"), _f32p), _ptr(res.get("err"), _f32p)]
        if owner is None:
            if m % (P * G):
                raise ValueError("contiguous segments need m % (P*G) == 0")
            rc = self.lib.echo_oracle_allreduce_ex(P, m, G, dtype, *args)
        else:
            owner = np.ascontiguousarray(owner, dtype=np.int32)
            if owner.shape != (ngroups,):
                raise ValueError("owner needs one rank per group")
            rc = self.lib.echo_oracle_allreduce_groups_ex(P, G, ngroups, _ptr(owner, _i32p),
                                                          dtype, *args)
        if rc != 0:
            raise ValueError(f"oracle allreduce failed ({rc})")
        return res


def contiguous_owner(P: int, n: int, G: int = 32) -> np.ndarray:
    """Owner rank of every group under the contiguous segment layout."""
    seg = n // P
    return (np.arange(n // G, dtype=np.int64) * G // seg).astype(np.int32)
