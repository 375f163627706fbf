"""Shared plumbing of the GPU parity tests: move seeded inputs to the device,
run the CUDA library through its C ABI, run the CPU oracle on the same bytes,
and compare everything bit for bit.

Comparisons (all exact):
  * stage-1 wire of every rank (packed codes and scale bytes),
  * the requantised wire (codes and scale bytes),
  * the output of every rank (bf16 or binary32 bit patterns),
  * the phase's fast and slow estimates (binary32 bit patterns).
"""
from __future__ import annotations

import numpy as np

from oracle.oracle import SENDER_EF, Params

G = 32


def torch():
    import torch as _t
    return _t


def to_device(x: np.ndarray):
    """(P, m) uint16 bf16 bits or float32 -> list of P device tensors."""
    t = torch()
    if x.dtype == np.uint16:
        base = t.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(t.bfloat16)
    else:
        base = t.from_numpy(np.ascontiguousarray(x)).cuda()
    return [base[r].clone() for r in range(x.shape[0])]


def from_device(tensors) -> np.ndarray:
    t = torch()
    stacked = t.stack([tt.reshape(-1) for tt in tensors])
    if stacked.dtype == t.bfloat16:
        return stacked.view(t.int16).cpu().numpy().view(np.uint16)
    return stacked.cpu().numpy()


def bits32(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def assert_same_bits(gpu, ref, what):
    gpu = np.asarray(gpu)
    ref = np.asarray(ref)
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    if gpu.dtype == np.float32:
        gpu, ref = bits32(gpu), bits32(ref)
    bad = np.flatnonzero(gpu.reshape(-1) != ref.reshape(-1))
    assert bad.size == 0, (f"{what}: {bad.size} mismatches, first at {bad[:8].tolist()}: "
                           f"gpu {gpu.reshape(-1)[bad[:4]].tolist()} oracle {ref.reshape(-1)[bad[:4]].tolist()}")


def params_tuple(p: Params):
    return (p.beta_fast, p.beta_slow, p.lam, p.enable)


class FullCompare:
    """One handle and the oracle side by side on a problem small enough to
    compare in full after every call.

    fused: run every call as the one-kernel path (True) or as the three
    pipelined kernels (False, the default here, so that the small problems
    these tests use keep covering the pipelined kernels; the one-kernel path
    has its own tests)."""

    def __init__(self, oracle, P, n, dtype: str, params: Params = Params(), variant: int = 0,
                 group: int = G, fused: bool = False):
        from bit_error_compensated_rank_b200 import echo
        self.echo = echo
        self.oracle = oracle
        self.P, self.n = P, n
        self.dtype = dtype
        self.params = params
        self.variant = variant
        self.group = group
        self.h = echo.Echo(P, n, echo.ECHO_BF16 if dtype == "bf16" else echo.ECHO_FP32, group)
        self.h.set_fused_limit(n if fused else 0)
        self.h.set_params(*params_tuple(params))
        if variant:
            self.h.set_variant(variant)
        self.state = {ph: (np.zeros(n, np.float32), np.zeros(n, np.float32)) for ph in (0, 1)}
        self.eps = {ph: np.zeros((P, n), np.float32) for ph in (0, 1)}

    def call(self, x: np.ndarray, phase: int = 0, out_of_place: bool = False,
             want_diag: bool = False):
        t = torch()
        assert x.shape == (self.P, self.n)
        dev = to_device(x)
        if out_of_place:
            recv = [t.empty_like(d) for d in dev]
            self.h.allreduce_out(dev, recv, phase)
        else:
            self.h.allreduce(dev, phase)
            recv = dev
        t.cuda.synchronize()
        f, s = self.state[phase]
        ref = self.oracle.allreduce(x, f, s, self.params, G=self.group, want_diag=want_diag,
                                    variant=self.variant, eps=self.eps[phase])
        got = from_device(recv)
        # no wait ran out; in the debug build also no bounds or guard failure
        assert self.h.device_status(clear=True) == 0, "device status"
        if out_of_place:  # the inputs are untouched
            assert_same_bits(from_device(dev), x, "send buffers")
        for r in range(self.P):
            codes, scales = self.h.get_wire(1, r)
            assert_same_bits(codes, ref["codes1"][r], f"stage-1 codes rank {r}")
            assert_same_bits(scales, ref["scales1"][r], f"stage-1 scales rank {r}")
        qc, qs = self.h.get_wire(2)
        assert_same_bits(qc, ref["qcodes"], "requantised codes")
        assert_same_bits(qs, ref["qscales"], "requantised scales")
        for r in range(self.P):
            assert_same_bits(got[r], ref["out"], f"output rank {r}")
        for ph in (0, 1):  # the called phase moved as the oracle's; the other did not move
            rf, rs = self.state[ph]
            gf, gs = self.h.get_state(ph)
            assert_same_bits(gf, rf, f"fast estimate phase {ph}")
            assert_same_bits(gs, rs, f"slow estimate phase {ph}")
            if self.variant & SENDER_EF:
                for r in range(self.P):
                    assert_same_bits(self.h.get_sender_state(ph, r), self.eps[ph][r],
                                     f"sender error rank {r} phase {ph}")
        return ref

    def close(self):
        self.h.close()


class SampledCompare:
    """Full-size problem, exact comparison on blocks of consecutive groups.

    Every output element depends only on its own group of every rank and on
    its own state, so running the oracle on the sampled groups alone (with
    each group's owner given explicitly) reproduces the full computation there
    exactly, call after call.
    """

    def __init__(self, oracle, P, n, dtype: str, params: Params = Params(), blocks=None,
                 block_groups: int = 64, seed: int = 0, variant: int = 0, group: int = G):
        from bit_error_compensated_rank_b200 import echo
        self.echo = echo
        self.oracle = oracle
        self.P, self.n, self.dtype, self.params = P, n, dtype, params
        self.group = group
        ngroups = n // group
        seg_groups = ngroups // P
        if blocks is None:
            starts = {0, max(0, ngroups - block_groups)}
            for s in range(1, P):  # both sides of every segment boundary
                starts.add(max(0, s * seg_groups - block_groups // 2))
            rng = np.random.default_rng(seed)
            for v in rng.integers(0, max(1, ngroups - block_groups), 6):
                starts.add(int(v))
            blocks = sorted(starts)
        bg = min(block_groups, ngroups)
        merged = []
        for b in blocks:
            b = min(b, ngroups - bg)
            if merged and b < merged[-1] + bg:
                continue
            merged.append(b)
        self.blocks = merged
        self.bg = bg
        self.groups = np.concatenate([np.arange(b, b + bg) for b in self.blocks])
        self.elems = (self.groups[:, None] * group + np.arange(group)[None, :]).reshape(-1)
        self.owner = (self.groups // seg_groups).astype(np.int32)
        self.h = echo.Echo(P, n, echo.ECHO_BF16 if dtype == "bf16" else echo.ECHO_FP32, group)
        self.h.set_params(*params_tuple(params))
        self.variant = variant
        if variant:
            self.h.set_variant(variant)
        m = self.elems.size
        self.state = {ph: (np.zeros(m, np.float32), np.zeros(m, np.float32)) for ph in (0, 1)}
        self.eps = {ph: np.zeros((P, m), np.float32) for ph in (0, 1)}
        self._idx = None

    def gather(self, tensors) -> np.ndarray:
        t = torch()
        if self._idx is None:
            self._idx = t.from_numpy(self.elems.astype(np.int64)).cuda()
        stacked = t.stack([tt.reshape(-1).index_select(0, self._idx) for tt in tensors])
        if stacked.dtype == t.bfloat16:
            return stacked.view(t.int16).cpu().numpy().view(np.uint16)
        return stacked.cpu().numpy()

    def call(self, tensors, phase: int = 0, stream=None):
        t = torch()
        x = self.gather(tensors)
        self.h.allreduce(tensors, phase, stream)
        t.cuda.synchronize()
        f, s = self.state[phase]
        G = self.group
        ref = self.oracle.allreduce(x, f, s, self.params, G=G, owner=self.owner,
                                    variant=self.variant, eps=self.eps[phase])
        got = self.gather(tensors)
        assert self.h.device_status(clear=True) == 0, "device status"
        for r in range(self.P):
            assert_same_bits(got[r], ref["out"], f"output rank {r}")
        half = G // 2
        for bi, b in enumerate(self.blocks):
            sl = slice(bi * self.bg, (bi + 1) * self.bg)
            csl = slice(bi * self.bg * half, (bi + 1) * self.bg * half)
            for r in range(self.P):
                codes, scales = self.h.get_wire_range(1, r, b, self.bg)
                assert_same_bits(codes, ref["codes1"][r][csl], f"stage-1 codes rank {r} block {b}")
                assert_same_bits(scales, ref["scales1"][r][sl], f"stage-1 scales rank {r} block {b}")
            qc, qs = self.h.get_wire_range(2, 0, b, self.bg)
            assert_same_bits(qc, ref["qcodes"][csl], f"requantised codes block {b}")
            assert_same_bits(qs, ref["qscales"][sl], f"requantised scales block {b}")
            esl = slice(bi * self.bg * G, (bi + 1) * self.bg * G)
            if self.params.enable:
                gf, gs = self.h.get_state_range(phase, b * G, self.bg * G)
                assert_same_bits(gf, f[esl], f"fast estimate block {b}")
                assert_same_bits(gs, s[esl], f"slow estimate block {b}")
            if self.variant & SENDER_EF:
                for r in range(self.P):
                    ge = self.h.get_sender_state(phase, r, b * G, self.bg * G)
                    assert_same_bits(ge, self.eps[phase][r][esl], f"sender error rank {r} block {b}")
        return ref

    def close(self):
        self.h.close()
