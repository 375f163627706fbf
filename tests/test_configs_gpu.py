"""The five workloads at their full sizes, CUDA path against the oracle.

1. P=2, one 4096-element bf16 partial per rank, 8 calls, seed 0 (full compare).
2. Qwen3-8B-shaped inference: P=4, 2048 tokens x 4096 hidden bf16, 72 calls,
   channel-scaled partials with 1 % outlier channels, forward state only.
3. Message-size sweep: P=8, 1 MiB .. 1 GiB bf16 per rank, N(0,1) with 0.1 %
   of values at 50x (the 1 GiB point is the benchmark's workload).
4. Llama-3-8B-shaped training step: P=4, 2 x 4096 tokens x 4096 hidden, 64
   forward calls then 64 backward calls (heavy-tailed gradients), separate
   state.
5. Deep residual stream: 256 layers, hidden 1024, 64 tokens, binary32, P=8,
   compensation on vs off vs the exact binary64 sum.

Large cases compare exactly on sampled blocks of groups (every segment
boundary, both ends, random blocks) after every call; see gpu_harness.
"""
import numpy as np
import pytest

from bit_error_compensated_rank_b200 import workloads as wl
from gpu_harness import FullCompare, SampledCompare
from oracle.oracle import Params

pytestmark = pytest.mark.gpu


def _bf16_buffers(P, n):
    import torch
    return [torch.empty(n, device="cuda", dtype=torch.bfloat16) for _ in range(P)]


def test_config1_two_ranks_4096(oracle):
    P, n = 2, 4096
    fc = FullCompare(oracle, P, n, "bf16")
    try:
        for k in range(8):
            fc.call(wl.gaussian(P, n, seed=0, call=k))
    finally:
        fc.close()


def test_config2_qwen3_8b_inference(oracle):
    import torch
    P, tokens, hidden, calls = 4, 2048, 4096, 72
    n = tokens * hidden
    sigma = torch.from_numpy(wl.channel_scale(hidden, seed=0)).cuda()
    sc = SampledCompare(oracle, P, n, "bf16")
    try:
        bufs = _bf16_buffers(P, n)
        for k in range(calls):
            for r in range(P):
                wl.torch_channel_scaled_(bufs[r], sigma, seed=0, call=k, rank=r)
            sc.call(bufs, phase=0)
        f, s = sc.h.get_state_range(1, 0, n)
        assert not f.any() and not s.any()  # backward state never touched
    finally:
        sc.close()


SWEEP = [1 << k for k in range(19, 30)]  # elements per rank: 1 MiB .. 1 GiB of bf16


@pytest.mark.parametrize("n", SWEEP, ids=[f"{(n * 2) >> 20}MiB" for n in SWEEP])
def test_config3_message_sweep(oracle, n):
    P = 8
    calls = 16 if n in (SWEEP[0], SWEEP[-1]) else 3
    sc = SampledCompare(oracle, P, n, "bf16")
    try:
        bufs = _bf16_buffers(P, n)
        for k in range(calls):
            for r in range(P):
                wl.torch_outlier_gaussian_(bufs[r], seed=0, call=k, rank=r)
            sc.call(bufs)
    finally:
        sc.close()


def test_config4_llama3_8b_training_step(oracle):
    import torch
    P, hidden = 4, 4096
    n = 2 * 4096 * hidden
    sigma = torch.from_numpy(wl.channel_scale(hidden, seed=1)).cuda()
    sc = SampledCompare(oracle, P, n, "bf16")
    try:
        bufs = _bf16_buffers(P, n)
        for k in range(64):
            for r in range(P):
                wl.torch_channel_scaled_(bufs[r], sigma, seed=1, call=k, rank=r)
            sc.call(bufs, phase=0)
        fwd_after = [a.copy() for a in sc.state[0]]
        for k in range(64):
            for r in range(P):
                wl.torch_student_t_(bufs[r], seed=1, call=k, rank=r)
            sc.call(bufs, phase=1)
        # backward calls left the forward state exactly as the forward pass left it
        for bi, b in enumerate(sc.blocks):
            esl = slice(bi * sc.bg * 32, (bi + 1) * sc.bg * 32)
            gf, gs = sc.h.get_state_range(0, b * 32, sc.bg * 32)
            assert (gf.view(np.uint32) == fwd_after[0][esl].view(np.uint32)).all()
            assert (gs.view(np.uint32) == fwd_after[1][esl].view(np.uint32)).all()
    finally:
        sc.close()


def _residual_partials(x, layer, P, hidden, seed):
    """Pre-norm tensor-parallel partials: (x / rms(x)) W_{layer,r} / sqrt(hidden * P)."""
    import torch
    xn = x / torch.sqrt(torch.mean(x.double() ** 2, dim=1, keepdim=True)).float()
    scale = 1.0 / float(np.sqrt(hidden * P))
    return [(xn @ wl.residual_weight(layer, r, hidden, seed, device=x.device)) * scale
            for r in range(P)]


def test_config5_deep_residual(oracle):
    """Bit-exact parity at every layer for both trajectories; the compensated
    sum of injected requantisation error stays within its closed-form bound
    (5 max|err|); and the compensated trajectory ends closer to the exact one."""
    import torch
    torch.backends.cuda.matmul.allow_tf32 = False
    P, hidden, tokens, layers, seed = 8, 1024, 64, 256, 0
    n = hidden * tokens
    x0 = torch.from_numpy(wl.residual_init(tokens, hidden, seed)).cuda()
    on = FullCompare(oracle, P, n, "fp32", Params())
    off = FullCompare(oracle, P, n, "fp32", Params(enable=False))
    x = {"on": x0.clone(), "off": x0.clone(), "ex": x0.clone()}
    D = np.zeros(n)
    emax = np.zeros(n)
    try:
        for layer in range(layers):
            pe = _residual_partials(x["ex"], layer, P, hidden, seed)
            x["ex"] = (x["ex"].double() + torch.stack(pe).double().sum(0)).float()
            for key, fc in (("on", on), ("off", off)):
                parts = torch.stack(_residual_partials(x[key], layer, P, hidden, seed))
                ref = fc.call(parts.reshape(P, n).cpu().numpy(), want_diag=(key == "on"))
                x[key] = x[key] + torch.from_numpy(ref["out"]).cuda().reshape(tokens, hidden)
                if key == "on":
                    D += ref["c"].astype(np.float64) - ref["err"].astype(np.float64)
                    emax = np.maximum(emax, np.abs(ref["err"].astype(np.float64)))
            assert (np.abs(D) <= 5 * emax * (1 + 1e-4) + 1e-30).all(), layer
        err_on = float(torch.linalg.norm(x["on"] - x["ex"]))
        err_off = float(torch.linalg.norm(x["off"] - x["ex"]))
        assert err_on < 0.9 * err_off, (err_on, err_off)
    finally:
        on.close()
        off.close()


@pytest.mark.parametrize("variant", [0, 3, 4], ids=["default", "owner_sum+sender_ef", "fp16_scale"])
def test_sixteen_ranks_large(oracle, variant):
    """The most ranks the library takes (P = 16) at 256 MiB of bf16 per rank,
    sampled blocks at every segment boundary, two calls."""
    import torch
    P, n = 16, 1 << 27
    sc = SampledCompare(oracle, P, n, "bf16", variant=variant, block_groups=32)
    try:
        bufs = _bf16_buffers(P, n)
        for k in range(2):
            for r in range(P):
                wl.torch_outlier_gaussian_(bufs[r], seed=44, call=k, rank=r)
            sc.call(bufs, phase=k)
    finally:
        sc.close()
        del bufs
        torch.cuda.empty_cache()
