"""Seeded synthetic inputs for the all-reduce workloads.

This module only draws random numbers and shapes them; it holds none of the
method's arithmetic, so both the CUDA path and the CPU oracle can be fed from
it. numpy generators serve the small cases (CPU), torch generators the large
ones (drawn directly on the device, then copied to the host only where a check
needs them).

Workloads (the shapes the Echo digests name: tensor-parallel partial sums of
Qwen3-8B and Llama-3-8B sized layers, a 1 GB message; see
[rit.work "Echo 4-bit GPU communication", section "When the gain changes the
infrastructure plan"]):

* ``gaussian``: i.i.d. N(0, 1) partials, fresh per call and rank.
* ``channel_scaled``: activations of a hidden-size-H layer; channel c has
  standard deviation sigma_c drawn once per run, log-uniform in [0.1, 1], and
  1 % of the channels are outliers at 20x.
* ``outlier_gaussian``: N(0, 1) with each value independently multiplied by 50
  with probability 0.001.
* ``student_t``: heavy-tailed gradients, scale * t_3, t_3 = Z / sqrt(chi2_3 / 3).
"""
from __future__ import annotations

import numpy as np

BF16 = "bf16"
FP32 = "fp32"


def seed_for(seed: int, *key: int) -> int:
    """A 63-bit seed derived from a base seed and integer key (call, rank, ...)."""
    ss = np.random.SeedSequence([int(seed)] + [int(k) for k in key])
    return int(ss.generate_state(2, dtype=np.uint64)[0] >> np.uint64(1))


def rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.default_rng(seed_for(seed, *key))


# --------------------------------------------------------------------------
# bf16 conversions (input preparation: bf16 is the upper half of binary32)
# --------------------------------------------------------------------------
def bf16_bits(a) -> np.ndarray:
    """binary32 -> bf16 bit patterns, rounding to nearest, halves to even."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lower = u & np.uint64(0xFFFF)
    upper = u >> np.uint64(16)
    round_up = (lower > 0x8000) | ((lower == 0x8000) & ((upper & np.uint64(1)) == 1))
    return (upper + round_up.astype(np.uint64)).astype(np.uint16)


def bf16_to_f32(bits) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _finish(v: np.ndarray, dtype: str) -> np.ndarray:
    v = v.astype(np.float32)
    return bf16_bits(v) if dtype == BF16 else v


# --------------------------------------------------------------------------
# numpy generators (CPU; tests and the oracle's baseline sample)
# --------------------------------------------------------------------------
def gaussian(P: int, n: int, seed: int, call: int, dtype: str = BF16) -> np.ndarray:
    """(P, n) i.i.d. N(0, 1) partials for one call."""
    out = np.empty((P, n), dtype=np.float32)
    for r in range(P):
        out[r] = rng(seed, 1, call, r).standard_normal(n, dtype=np.float32)
    return _finish(out, dtype)


def channel_scale(hidden: int, seed: int, outlier_frac: float = 0.01,
                  outlier_mult: float = 20.0) -> np.ndarray:
    """Per-channel standard deviation: log-uniform in [0.1, 1], a fixed 1 % of
    channels multiplied by 20. Drawn once per run."""
    g = rng(seed, 2)
    sigma = np.exp(g.uniform(np.log(0.1), np.log(1.0), hidden)).astype(np.float32)
    k = int(round(outlier_frac * hidden))
    idx = g.choice(hidden, size=k, replace=False)
    sigma[idx] *= np.float32(outlier_mult)
    return sigma


def channel_scaled(P: int, tokens: int, hidden: int, sigma: np.ndarray, seed: int,
                   call: int, dtype: str = BF16) -> np.ndarray:
    """(P, tokens*hidden) partials, element (t, c) ~ sigma_c * N(0, 1)."""
    out = np.empty((P, tokens * hidden), dtype=np.float32)
    for r in range(P):
        z = rng(seed, 3, call, r).standard_normal((tokens, hidden), dtype=np.float32)
        out[r] = (z * sigma[None, :]).reshape(-1)
    return _finish(out, dtype)


def outlier_gaussian(P: int, n: int, seed: int, call: int, p: float = 1e-3,
                     mult: float = 50.0, dtype: str = BF16) -> np.ndarray:
    out = np.empty((P, n), dtype=np.float32)
    for r in range(P):
        g = rng(seed, 4, call, r)
        z = g.standard_normal(n, dtype=np.float32)
        hit = g.random(n) < p
        z[hit] *= np.float32(mult)
        out[r] = z
    return _finish(out, dtype)


def student_t(P: int, n: int, seed: int, call: int, nu: int = 3, scale: float = 1e-3,
              dtype: str = BF16) -> np.ndarray:
    out = np.empty((P, n), dtype=np.float32)
    for r in range(P):
        g = rng(seed, 5, call, r)
        z = g.standard_normal(n)
        chi2 = g.chisquare(nu, n)
        out[r] = (scale * z / np.sqrt(chi2 / nu)).astype(np.float32)
    return _finish(out, dtype)


# --------------------------------------------------------------------------
# torch generators (device-resident inputs for the large cases)
# --------------------------------------------------------------------------
def _torch_gen(device, seed: int, *key: int):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed_for(seed, *key))
    return g


def torch_gaussian_(buf, seed: int, call: int, rank: int):
    """Fill a device tensor (any float dtype) with N(0, 1) in place."""
    import torch
    g = _torch_gen(buf.device, seed, 11, call, rank)
    tmp = torch.randn(buf.shape, generator=g, device=buf.device, dtype=torch.float32)
    buf.copy_(tmp)
    return buf


def torch_outlier_gaussian_(buf, seed: int, call: int, rank: int, p: float = 1e-3,
                            mult: float = 50.0, chunk: int = 1 << 26):
    """N(0, 1) with 0.1 % of values at 50x, generated chunk by chunk on the
    device so a 1 GiB message needs no full-size float32 temporary."""
    import torch
    flat = buf.view(-1)
    g = _torch_gen(buf.device, seed, 14, call, rank)
    for a in range(0, flat.numel(), chunk):
        b = min(flat.numel(), a + chunk)
        z = torch.randn(b - a, generator=g, device=buf.device, dtype=torch.float32)
        u = torch.rand(b - a, generator=g, device=buf.device, dtype=torch.float32)
        z = torch.where(u < p, z * mult, z)
        flat[a:b].copy_(z)
    return buf


def torch_channel_scaled_(buf, sigma, seed: int, call: int, rank: int):
    """buf viewed as (tokens, hidden): element (t, c) ~ sigma_c * N(0, 1)."""
    import torch
    hidden = sigma.numel()
    g = _torch_gen(buf.device, seed, 13, call, rank)
    z = torch.randn(buf.numel() // hidden, hidden, generator=g, device=buf.device,
                    dtype=torch.float32)
    buf.view(-1, hidden).copy_(z * sigma[None, :])
    return buf


def torch_student_t_(buf, seed: int, call: int, rank: int, nu: int = 3,
                     scale: float = 1e-3):
    import torch
    g = _torch_gen(buf.device, seed, 15, call, rank)
    z = torch.randn(buf.shape, generator=g, device=buf.device, dtype=torch.float32)
    # chi-square with nu degrees of freedom as a sum of nu squared normals
    chi2 = torch.zeros_like(z)
    for _ in range(nu):
        w = torch.randn(buf.shape, generator=g, device=buf.device, dtype=torch.float32)
        chi2 += w * w
    buf.copy_(scale * z / torch.sqrt(chi2 / nu))
    return buf


# --------------------------------------------------------------------------
# deep residual stream (pre-norm form)
# --------------------------------------------------------------------------
def residual_weight(layer: int, rank: int, hidden: int, seed: int, device=None):
    """W_{layer,rank} with i.i.d. N(0, 1) entries, seeded per (layer, rank)."""
    if device is None:
        return rng(seed, 6, layer, rank).standard_normal((hidden, hidden), dtype=np.float32)
    import torch
    g = _torch_gen(device, seed, 16, layer, rank)
    return torch.randn(hidden, hidden, generator=g, device=device, dtype=torch.float32)


def residual_init(tokens: int, hidden: int, seed: int) -> np.ndarray:
    return rng(seed, 7).standard_normal((tokens, hidden), dtype=np.float32)
