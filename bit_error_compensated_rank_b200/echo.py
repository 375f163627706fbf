"""ctypes binding of ``libecho.so`` (the C ABI in ``include/echo.h``).

Functions keep the C names and only marshal arguments: every step of the
all-reduce runs in the library's CUDA kernels. There is no fallback: importing
this module raises ``ImportError`` when the library has not been built, and
every failing call raises :class:`EchoError` with the library's message.

Device buffers are passed as integer addresses; the helpers that take torch
tensors read ``data_ptr()`` and the current stream's handle, nothing more.

``ECHO_LIB=debug`` in the environment loads the debug build
(``libecho_debug.so``: device-side bounds checks and guard bytes, reported in
the device status word) instead of the release build.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib",
                        "libecho_debug.so" if os.environ.get("ECHO_LIB") == "debug" else "libecho.so")

ECHO_BF16 = 0
ECHO_FP32 = 1
ECHO_FWD = 0
ECHO_BWD = 1
ECHO_OK = 0
ECHO_ERR_INVALID = -1
ECHO_ERR_UNSUPPORTED = -2
ECHO_ERR_CUDA = -3
ECHO_ERR_OOM = -4
ECHO_MAX_RANKS = 16
ECHO_GROUP = 32
ECHO_VARIANT_OWNER_SUM = 1
ECHO_VARIANT_SENDER_EF = 2
ECHO_VARIANT_FP16_SCALE = 4
ECHO_STATUS_TIMEOUT_K1 = 1
ECHO_STATUS_TIMEOUT_K2 = 2
ECHO_STATUS_TIMEOUT_K3 = 4
ECHO_STATUS_BOUNDS = 8
ECHO_STATUS_CANARY = 16

EXPORTED = (
    "echo_create", "echo_allreduce", "echo_allreduce_out", "echo_allreduce_host",
    "echo_reset", "echo_destroy", "echo_last_error", "echo_last_status", "echo_set_params",
    "echo_get_state", "echo_set_state", "echo_get_state_range", "echo_get_wire",
    "echo_get_wire_range", "echo_stats", "echo_model_bytes", "echo_set_timing",
    "echo_last_kernel_ms", "echo_kernel_ms_total", "echo_device_status",
    "echo_allreduce_static", "echo_static_status", "echo_set_variant", "echo_get_sender_state", "echo_set_sender_state",
    "echo_set_fused_limit", "echo_get_fused_limit",
    "echo_model_bytes_ex", "echo_debug_build", "echo_debug_touch_guard",
    "echo_dist_create", "echo_dist_export", "echo_dist_connect", "echo_dist_stage",
    "echo_dist_set_params", "echo_dist_set_variant", "echo_dist_get_state",
    "echo_dist_device_status", "echo_dist_destroy",
)
ECHO_DIST_HANDLE_BYTES = 320

_vp = ctypes.c_void_p
_sz = ctypes.c_size_t
_int = ctypes.c_int
_f32p = ctypes.POINTER(ctypes.c_float)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_u64p = ctypes.POINTER(ctypes.c_uint64)
_vpp = ctypes.POINTER(ctypes.c_void_p)


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m bit_error_compensated_rank_b200.build`"
            " (the CUDA library is the only implementation; there is no fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    sig = {
        "echo_create": (_vp, [_int, _sz, _int, _int]),
        "echo_allreduce": (_int, [_vp, _vpp, _int, _vp]),
        "echo_allreduce_out": (_int, [_vp, _vpp, _vpp, _int, _vp]),
        "echo_allreduce_host": (_int, [_vp, _vpp, _vp, _int, _vp]),
        "echo_reset": (_int, [_vp, _int]),
        "echo_destroy": (_int, [_vp]),
        "echo_last_error": (ctypes.c_char_p, []),
        "echo_last_status": (_int, []),
        "echo_set_params": (_int, [_vp, ctypes.c_float, ctypes.c_float, ctypes.c_float, _int]),
        "echo_get_state": (_int, [_vp, _int, _f32p, _f32p]),
        "echo_set_state": (_int, [_vp, _int, _f32p, _f32p]),
        "echo_get_state_range": (_int, [_vp, _int, _sz, _sz, _f32p, _f32p]),
        "echo_get_wire": (_int, [_vp, _int, _int, _u8p, _u8p]),
        "echo_get_wire_range": (_int, [_vp, _int, _int, _sz, _sz, _u8p, _u8p]),
        "echo_stats": (_int, [_vp, _u64p, _u64p, _u64p]),
        "echo_model_bytes": (_int, [_int, _sz, _int, _int, _u64p]),
        "echo_set_timing": (_int, [_vp, _int]),
        "echo_last_kernel_ms": (_int, [_vp, _f32p]),
        "echo_kernel_ms_total": (_int, [_vp, ctypes.POINTER(ctypes.c_double), _u64p]),
        "echo_device_status": (_int, [_vp, ctypes.POINTER(ctypes.c_int), _int]),
        "echo_allreduce_static": (_int, [_int, _sz, _int, _vpp, _vp, _vp, ctypes.c_float, ctypes.c_float,
                                         ctypes.c_float, _int, _vp]),
        "echo_static_status": (_int, [ctypes.POINTER(ctypes.c_int), _int]),
        "echo_set_variant": (_int, [_vp, _int]),
        "echo_set_fused_limit": (_int, [_vp, _sz]),
        "echo_get_fused_limit": (_int, [_vp, ctypes.POINTER(ctypes.c_size_t)]),
        "echo_get_sender_state": (_int, [_vp, _int, _int, _sz, _sz, _f32p]),
        "echo_set_sender_state": (_int, [_vp, _int, _int, _f32p]),
        "echo_model_bytes_ex": (_int, [_int, _sz, _int, _int, _int, _int, _u64p]),
        "echo_debug_build": (_int, []),
        "echo_debug_touch_guard": (_int, [_vp]),
        "echo_dist_create": (_vp, [_int, _int, _sz, _int, _int]),
        "echo_dist_export": (_int, [_vp, _u8p]),
        "echo_dist_connect": (_int, [_vp, _u8p]),
        "echo_dist_stage": (_int, [_vp, _int, _vp, _vp, _int, _vp]),
        "echo_dist_set_params": (_int, [_vp, ctypes.c_float, ctypes.c_float, ctypes.c_float, _int]),
        "echo_dist_set_variant": (_int, [_vp, _int]),
        "echo_dist_get_state": (_int, [_vp, _int, _f32p, _f32p]),
        "echo_dist_device_status": (_int, [_vp, ctypes.POINTER(ctypes.c_int), _int]),
        "echo_dist_destroy": (_int, [_vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


class EchoError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"echo error {code}: {message}")
        self.code = code


def echo_last_error() -> str:
    return (_lib.echo_last_error() or b"").decode()


def echo_last_status() -> int:
    return _lib.echo_last_status()


def _check(rc: int) -> None:
    if rc != ECHO_OK:
        raise EchoError(rc, echo_last_error())


def _ptr_array(ptrs) -> ctypes.Array:
    return (ctypes.c_void_p * len(ptrs))(*[int(p) for p in ptrs])


def _np(a, ctype):
    return None if a is None else a.ctypes.data_as(ctype)


# ---- the C entry points, one to one --------------------------------------
def echo_create(P: int, n: int, group: int = ECHO_GROUP, dtype: int = ECHO_BF16) -> int:
    h = _lib.echo_create(P, n, group, dtype)
    if not h:
        raise EchoError(_lib.echo_last_status(), echo_last_error())
    return h


def echo_allreduce(h: int, rank_ptrs, phase: int = ECHO_FWD, stream: int = 0) -> None:
    _check(_lib.echo_allreduce(h, _ptr_array(rank_ptrs), phase, stream))


def echo_allreduce_out(h: int, send_ptrs, recv_ptrs, phase: int = ECHO_FWD, stream: int = 0) -> None:
    _check(_lib.echo_allreduce_out(h, _ptr_array(send_ptrs), _ptr_array(recv_ptrs), phase, stream))


def echo_allreduce_host(h: int, host_send_ptrs, host_recv_ptr: int, phase: int = ECHO_FWD,
                        stream: int = 0) -> None:
    _check(_lib.echo_allreduce_host(h, _ptr_array(host_send_ptrs), host_recv_ptr, phase, stream))


def echo_allreduce_static(P: int, n: int, dtype: int, rank_ptrs, f_ptr: int, s_ptr: int,
                          beta_fast: float = 0.5, beta_slow: float = 0.875, lam: float = 0.5,
                          enable: bool = True, stream: int = 0) -> None:
    """The all-reduce without device allocation (see include/echo.h): the
    caller passes the rank buffers and this phase's state arrays f, s."""
    _check(_lib.echo_allreduce_static(P, n, dtype, _ptr_array(rank_ptrs), f_ptr, s_ptr, beta_fast,
                                      beta_slow, lam, int(bool(enable)), stream))


def echo_static_status(clear: bool = False) -> int:
    """The static path's device status word on the current device (waits for
    the device); ``clear`` zeroes it after reading."""
    st = ctypes.c_int(0)
    _check(_lib.echo_static_status(ctypes.byref(st), int(bool(clear))))
    return st.value


def echo_reset(h: int, phase_mask: int = 3) -> None:
    _check(_lib.echo_reset(h, phase_mask))


def echo_destroy(h: int) -> None:
    _check(_lib.echo_destroy(h))


def echo_set_params(h: int, beta_fast: float = 0.5, beta_slow: float = 0.875, lam: float = 0.5,
                    enable: bool = True) -> None:
    _check(_lib.echo_set_params(h, beta_fast, beta_slow, lam, int(bool(enable))))


def echo_get_state(h: int, phase: int, n: int) -> tuple[np.ndarray, np.ndarray]:
    f = np.empty(n, np.float32)
    s = np.empty(n, np.float32)
    _check(_lib.echo_get_state(h, phase, _np(f, _f32p), _np(s, _f32p)))
    return f, s


def echo_set_state(h: int, phase: int, f: np.ndarray, s: np.ndarray) -> None:
    f = np.ascontiguousarray(f, np.float32)
    s = np.ascontiguousarray(s, np.float32)
    _check(_lib.echo_set_state(h, phase, _np(f, _f32p), _np(s, _f32p)))


def echo_get_state_range(h: int, phase: int, offset: int, count: int):
    f = np.empty(count, np.float32)
    s = np.empty(count, np.float32)
    _check(_lib.echo_get_state_range(h, phase, offset, count, _np(f, _f32p), _np(s, _f32p)))
    return f, s


def echo_get_wire(h: int, stage: int, rank: int, n: int, group: int = ECHO_GROUP,
                  fp16_scale: bool = False):
    """Codes (uint8) and scales: uint8 bytes, or uint16 binary16 patterns
    when the handle runs ECHO_VARIANT_FP16_SCALE (say so with fp16_scale)."""
    codes = np.empty(n // 2, np.uint8)
    scales = np.empty(n // group, np.uint16 if fp16_scale else np.uint8)
    _check(_lib.echo_get_wire(h, stage, rank, _np(codes, _u8p), _np(scales, _u8p)))
    return codes, scales


def echo_get_wire_range(h: int, stage: int, rank: int, group_offset: int, ngroups: int,
                        group: int = ECHO_GROUP, fp16_scale: bool = False):
    codes = np.empty(ngroups * group // 2, np.uint8)
    scales = np.empty(ngroups, np.uint16 if fp16_scale else np.uint8)
    _check(_lib.echo_get_wire_range(h, stage, rank, group_offset, ngroups,
                                    _np(codes, _u8p), _np(scales, _u8p)))
    return codes, scales


def echo_stats(h: int) -> dict:
    link, hbm, calls = ctypes.c_uint64(), ctypes.c_uint64(), ctypes.c_uint64()
    _check(_lib.echo_stats(h, ctypes.byref(link), ctypes.byref(hbm), ctypes.byref(calls)))
    return {"link_bytes": link.value, "model_hbm_bytes": hbm.value, "calls": calls.value}


def echo_model_bytes(P: int, n: int, dtype: int = ECHO_BF16, enable: bool = True) -> dict:
    out = (ctypes.c_uint64 * 4)()
    _check(_lib.echo_model_bytes(P, n, dtype, int(bool(enable)), out))
    return {"k1": out[0], "k2": out[1], "k3": out[2], "link": out[3],
            "total": out[0] + out[1] + out[2]}


def echo_debug_build() -> bool:
    return bool(_lib.echo_debug_build())


def echo_debug_touch_guard(h: int) -> None:
    _check(_lib.echo_debug_touch_guard(h))


def echo_model_bytes_ex(P: int, n: int, group: int = ECHO_GROUP, dtype: int = ECHO_BF16,
                        enable: bool = True, variant: int = 0) -> dict:
    out = (ctypes.c_uint64 * 4)()
    _check(_lib.echo_model_bytes_ex(P, n, group, dtype, int(bool(enable)), variant, out))
    return {"k1": out[0], "k2": out[1], "k3": out[2], "link": out[3],
            "total": out[0] + out[1] + out[2]}


def echo_set_variant(h: int, variant: int) -> None:
    _check(_lib.echo_set_variant(h, variant))


def echo_set_fused_limit(h: int, max_n: int) -> None:
    _check(_lib.echo_set_fused_limit(h, max_n))


def echo_get_fused_limit(h: int) -> int:
    v = ctypes.c_size_t()
    _check(_lib.echo_get_fused_limit(h, ctypes.byref(v)))
    return v.value


def echo_get_sender_state(h: int, phase: int, rank: int, offset: int, count: int) -> np.ndarray:
    out = np.empty(count, np.float32)
    _check(_lib.echo_get_sender_state(h, phase, rank, offset, count, _np(out, _f32p)))
    return out


def echo_set_sender_state(h: int, phase: int, rank: int, values: np.ndarray) -> None:
    values = np.ascontiguousarray(values, np.float32)
    _check(_lib.echo_set_sender_state(h, phase, rank, _np(values, _f32p)))


def echo_set_timing(h: int, enable: bool = True) -> None:
    _check(_lib.echo_set_timing(h, int(bool(enable))))


def echo_last_kernel_ms(h: int) -> list[float]:
    ms = (ctypes.c_float * 3)()
    _check(_lib.echo_last_kernel_ms(h, ms))
    return [ms[0], ms[1], ms[2]]


def echo_device_status(h: int, clear: bool = False) -> int:
    st = ctypes.c_int()
    _check(_lib.echo_device_status(h, ctypes.byref(st), int(bool(clear))))
    return st.value


def echo_kernel_ms_total(h: int) -> tuple[list[float], int]:
    ms = (ctypes.c_double * 3)()
    calls = ctypes.c_uint64()
    _check(_lib.echo_kernel_ms_total(h, ms, ctypes.byref(calls)))
    return [ms[0], ms[1], ms[2]], calls.value


# ---- torch conveniences (plumbing only) -----------------------------------
def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return ECHO_BF16
    if t.dtype == torch.float32:
        return ECHO_FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream(stream) -> int:
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


class Echo:
    """Owning wrapper of one handle: ``Echo(P, n, dtype)``; call
    :meth:`allreduce` with P device tensors (torch) of n elements each."""

    def __init__(self, P: int, n: int, dtype: int = ECHO_BF16, group: int = ECHO_GROUP):
        self.P, self.n, self.dtype, self.group = P, n, dtype, group
        self.variant = 0
        self._arrays = {}
        self.h = echo_create(P, n, group, dtype)

    def _ptrs(self, tensors) -> ctypes.Array:
        """The tensors' device addresses as a C array, kept for reuse: a
        layer that reduces the same buffers every step pays the marshalling
        once. The C ABI sees plain pointers and cannot know a buffer's size,
        so a new set of tensors is checked here first: P contiguous CUDA
        tensors of the handle's dtype with at least n elements each."""
        key = tuple((t.data_ptr(), t.numel(), t.dtype) for t in tensors)
        arr = self._arrays.get(key)
        if arr is None:
            self._check_tensors(tensors)
            if len(self._arrays) >= 64:
                self._arrays.clear()
            arr = self._arrays[key] = _ptr_array([k[0] for k in key])
        return arr

    def _check_tensors(self, tensors) -> None:
        if len(tensors) != self.P:
            raise EchoError(ECHO_ERR_INVALID, f"{len(tensors)} tensors for P = {self.P} ranks")
        for r, t in enumerate(tensors):
            if not t.is_cuda or not t.is_contiguous():
                raise EchoError(ECHO_ERR_INVALID, f"rank {r}: tensor must be a contiguous CUDA tensor")
            if _dtype_code(t) != self.dtype:
                raise EchoError(ECHO_ERR_INVALID, f"rank {r}: dtype {t.dtype} does not match the handle")
            if t.numel() < self.n:
                raise EchoError(ECHO_ERR_INVALID, f"rank {r}: {t.numel()} elements, the handle needs {self.n}")

    def allreduce(self, tensors, phase: int = ECHO_FWD, stream=None) -> None:
        _check(_lib.echo_allreduce(self.h, self._ptrs(tensors), phase, _stream(stream)))

    def allreduce_out(self, send, recv, phase: int = ECHO_FWD, stream=None) -> None:
        _check(_lib.echo_allreduce_out(self.h, self._ptrs(send), self._ptrs(recv), phase,
                                       _stream(stream)))

    def allreduce_host(self, host_send, host_recv, phase: int = ECHO_FWD, stream=None) -> None:
        if len(host_send) != self.P:
            raise EchoError(ECHO_ERR_INVALID, f"{len(host_send)} tensors for P = {self.P} ranks")
        for t in list(host_send) + [host_recv]:
            if t.is_cuda or not t.is_contiguous() or _dtype_code(t) != self.dtype or t.numel() < self.n:
                raise EchoError(ECHO_ERR_INVALID, "host tensors must be contiguous CPU tensors of the "
                                                  f"handle's dtype with at least {self.n} elements")
        echo_allreduce_host(self.h, [t.data_ptr() for t in host_send], host_recv.data_ptr(),
                            phase, _stream(stream))

    def set_params(self, beta_fast=0.5, beta_slow=0.875, lam=0.5, enable=True) -> None:
        echo_set_params(self.h, beta_fast, beta_slow, lam, enable)

    def reset(self, phase_mask: int = 3) -> None:
        echo_reset(self.h, phase_mask)

    def set_variant(self, variant: int) -> None:
        echo_set_variant(self.h, variant)
        self.variant = variant

    def set_fused_limit(self, max_n: int) -> None:
        """Calls with n <= max_n run as one kernel (0: never)."""
        echo_set_fused_limit(self.h, max_n)

    def fused_limit(self) -> int:
        return echo_get_fused_limit(self.h)

    def get_sender_state(self, phase: int, rank: int, offset: int = 0, count: int | None = None):
        return echo_get_sender_state(self.h, phase, rank, offset, self.n - offset if count is None else count)

    def set_sender_state(self, phase: int, rank: int, values) -> None:
        echo_set_sender_state(self.h, phase, rank, values)

    def get_state(self, phase: int = ECHO_FWD):
        return echo_get_state(self.h, phase, self.n)

    def set_state(self, phase: int, f, s) -> None:
        echo_set_state(self.h, phase, f, s)

    def get_state_range(self, phase: int, offset: int, count: int):
        return echo_get_state_range(self.h, phase, offset, count)

    def get_wire(self, stage: int, rank: int = 0):
        return echo_get_wire(self.h, stage, rank, self.n, self.group,
                             bool(self.variant & ECHO_VARIANT_FP16_SCALE))

    def get_wire_range(self, stage: int, rank: int, group_offset: int, ngroups: int):
        return echo_get_wire_range(self.h, stage, rank, group_offset, ngroups, self.group,
                                   bool(self.variant & ECHO_VARIANT_FP16_SCALE))

    def stats(self) -> dict:
        return echo_stats(self.h)

    def set_timing(self, enable: bool = True) -> None:
        echo_set_timing(self.h, enable)

    def last_kernel_ms(self) -> list[float]:
        return echo_last_kernel_ms(self.h)

    def kernel_ms_total(self) -> tuple[list[float], int]:
        return echo_kernel_ms_total(self.h)

    def device_status(self, clear: bool = False) -> int:
        return echo_device_status(self.h, clear)

    def debug_touch_guard(self) -> None:
        echo_debug_touch_guard(self.h)

    def close(self) -> None:
        if self.h:
            echo_destroy(self.h)
            self.h = None

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ---- one rank per handle (several processes, or several ranks per process) ----
def dist_allreduce(handles, xs, outs, barrier, phase: int = ECHO_FWD, stream=None, sync: bool = False) -> None:
    """One call of the ranks ``handles`` held by this process (one or more),
    with their partials ``xs`` and outputs ``outs``: every local rank's stage
    1, ``barrier()``, every local rank's stage 2, ``barrier()``, every local
    rank's stage 3. The library orders the stages on the GPU with events;
    the two barriers only make sure every rank, in every process, has enqueued
    a stage before any enqueues the next, so the host never waits for the
    GPU. ``sync=True`` is the host-ordered form kept for comparison: it waits
    for the stream before each barrier and adds one after stage 3."""
    import torch
    st = stream if stream is not None else torch.cuda.current_stream()
    for k in (1, 2, 3):
        for d, x, out in zip(handles, xs, outs):
            d.stage(k, x, out, phase, st)
        if sync:
            st.synchronize()
        if k < 3 or sync:
            barrier()


class DistEcho:
    """One rank of an all-reduce whose ranks are separate handles (the
    echo_dist_* entry points): ``DistEcho(world, rank, n, dtype)``, exchange
    the blobs (``export`` on every rank, then ``connect`` with all of them in
    rank order), then :meth:`allreduce`. ``barrier`` is a callable that
    returns when every rank has called it (``torch.distributed.barrier`` on a
    gloo group, in practice)."""

    def __init__(self, world: int, rank: int, n: int, dtype: int = ECHO_BF16, group: int = ECHO_GROUP):
        self.world, self.rank, self.n, self.dtype, self.group = world, rank, n, dtype, group
        self.seg = n // world
        h = _lib.echo_dist_create(world, rank, n, group, dtype)
        if not h:
            raise EchoError(_lib.echo_last_status(), echo_last_error())
        self.h = h

    def export(self) -> bytes:
        buf = (ctypes.c_uint8 * ECHO_DIST_HANDLE_BYTES)()
        _check(_lib.echo_dist_export(self.h, buf))
        return bytes(buf)

    def connect(self, handles) -> None:
        if len(handles) != self.world or any(len(b) != ECHO_DIST_HANDLE_BYTES for b in handles):
            raise EchoError(ECHO_ERR_INVALID, f"need {self.world} blobs of {ECHO_DIST_HANDLE_BYTES} bytes")
        blob = (ctypes.c_uint8 * (self.world * ECHO_DIST_HANDLE_BYTES)).from_buffer_copy(b"".join(handles))
        _check(_lib.echo_dist_connect(self.h, blob))

    def _check_tensor(self, t, what: str) -> None:
        if not t.is_cuda or not t.is_contiguous() or _dtype_code(t) != self.dtype or t.numel() < self.n:
            raise EchoError(ECHO_ERR_INVALID, f"{what}: a contiguous CUDA tensor of the handle's dtype "
                                              f"with at least {self.n} elements is needed")

    def stage(self, stage: int, x=None, out=None, phase: int = ECHO_FWD, stream=None) -> None:
        if stage == 1:
            self._check_tensor(x, "x")
        if stage == 3:
            self._check_tensor(out, "out")
        _check(_lib.echo_dist_stage(self.h, stage, x.data_ptr() if stage == 1 else None,
                                    out.data_ptr() if stage == 3 else None, phase, _stream(stream)))

    def allreduce(self, x, out, barrier, phase: int = ECHO_FWD, stream=None, sync: bool = False) -> None:
        """One call of this rank (see :func:`dist_allreduce`)."""
        dist_allreduce([self], [x], [out], barrier, phase, stream, sync)

    def set_params(self, beta_fast=0.5, beta_slow=0.875, lam=0.5, enable=True) -> None:
        _check(_lib.echo_dist_set_params(self.h, beta_fast, beta_slow, lam, int(bool(enable))))

    def set_variant(self, variant: int) -> None:
        _check(_lib.echo_dist_set_variant(self.h, variant))

    def get_state(self, phase: int = ECHO_FWD):
        f = np.empty(self.seg, np.float32)
        s = np.empty(self.seg, np.float32)
        _check(_lib.echo_dist_get_state(self.h, phase, _np(f, _f32p), _np(s, _f32p)))
        return f, s

    def device_status(self, clear: bool = False) -> int:
        st = ctypes.c_int()
        _check(_lib.echo_dist_device_status(self.h, ctypes.byref(st), int(bool(clear))))
        return st.value

    def close(self) -> None:
        if self.h:
            _check(_lib.echo_dist_destroy(self.h))
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
