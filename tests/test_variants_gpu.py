"""The two variants of where the rounding errors are fed back, CUDA path
against the oracle bit for bit: the correction folded into the owner's sum
(ECHO_VARIANT_OWNER_SUM) and sender-side feedback of every rank's own
rounding-#1 error (ECHO_VARIANT_SENDER_EF), alone and together.

Compared after every call: both wires, every rank's output, both phases' f
and s, and every rank's sender error."""
import numpy as np
import pytest

from bit_error_compensated_rank_b200 import workloads as wl
from bit_error_compensated_rank_b200.workloads import gaussian, outlier_gaussian
from gpu_harness import FullCompare, SampledCompare, assert_same_bits
from oracle.oracle import OWNER_SUM, SENDER_EF, Params

pytestmark = pytest.mark.gpu

VARIANTS = [OWNER_SUM, SENDER_EF, OWNER_SUM | SENDER_EF]
VIDS = ["owner_sum", "sender_ef", "both"]


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("P,n", [(2, 2 * 32 * 37), (8, 8 * 32 * 301), (16, 16 * 32 * 33), (5, 5 * 32)])
@pytest.mark.parametrize("variant", VARIANTS, ids=VIDS)
def test_variant_sequences(oracle, variant, P, n, dtype):
    fc = FullCompare(oracle, P, n, dtype, variant=variant)
    try:
        for k, ph in enumerate([0, 0, 1, 0, 1, 1]):
            x = outlier_gaussian(P, n, seed=50 + P, call=k, dtype=dtype)
            fc.call(x, phase=ph)
    finally:
        fc.close()


def test_sender_feedback_without_owner_correction(oracle):
    P, n = 4, 4 * 32 * 129
    fc = FullCompare(oracle, P, n, "bf16", params=Params(enable=False), variant=SENDER_EF)
    try:
        for k in range(4):
            fc.call(gaussian(P, n, seed=3, call=k))
    finally:
        fc.close()


def test_switching_variants_carries_state(oracle):
    """State written under one variant is read under the next; the sender
    errors start at zero when sender feedback is first switched on."""
    P, n = 4, 4 * 32 * 100
    fc = FullCompare(oracle, P, n, "bf16")
    try:
        plan = [0, 0, OWNER_SUM, OWNER_SUM | SENDER_EF, SENDER_EF, 0, OWNER_SUM]
        for k, variant in enumerate(plan):
            if variant != fc.variant:
                fc.h.set_variant(variant)
                fc.variant = variant
            fc.call(gaussian(P, n, seed=9, call=k))
    finally:
        fc.close()


def test_sender_state_checkpoint_and_reset(oracle):
    P, n = 4, 4 * 32 * 64
    fc = FullCompare(oracle, P, n, "bf16", variant=SENDER_EF)
    try:
        fc.call(gaussian(P, n, seed=4, call=0))
        g = np.random.default_rng(1)
        for r in range(P):
            e = (g.standard_normal(n) * 0.01).astype(np.float32)
            fc.h.set_sender_state(0, r, e)
            assert_same_bits(fc.h.get_sender_state(0, r), e, "sender state round trip")
            fc.eps[0][r] = e
        fc.call(gaussian(P, n, seed=4, call=1))
        fc.h.reset(1)
        for r in range(P):
            assert not fc.h.get_sender_state(0, r).any()
    finally:
        fc.close()


def test_variant_bytes_model():
    from bit_error_compensated_rank_b200 import echo
    P, n = 8, 1 << 29
    base = echo.echo_model_bytes_ex(P, n, echo.ECHO_GROUP, echo.ECHO_BF16, True, 0)
    osum = echo.echo_model_bytes_ex(P, n, echo.ECHO_GROUP, echo.ECHO_BF16, True, OWNER_SUM)
    ef = echo.echo_model_bytes_ex(P, n, echo.ECHO_GROUP, echo.ECHO_BF16, True, SENDER_EF)
    assert base == echo.echo_model_bytes(P, n, echo.ECHO_BF16, True)
    assert base["total"] - osum["total"] == 8 * n
    assert ef["total"] - base["total"] == 8 * P * n


@pytest.mark.parametrize("variant", VARIANTS, ids=VIDS)
def test_variant_at_one_gib(oracle, variant):
    """The benchmark's size (P = 8, 1 GiB bf16 per rank), sampled blocks."""
    P, n = 8, 1 << 29
    sc = SampledCompare(oracle, P, n, "bf16", variant=variant)
    try:
        import torch
        bufs = [torch.empty(n, device="cuda", dtype=torch.bfloat16) for _ in range(P)]
        for k in range(3):
            for r in range(P):
                wl.torch_outlier_gaussian_(bufs[r], seed=7, call=k, rank=r)
            sc.call(bufs)
    finally:
        sc.close()


def test_full_compensation_stops_error_growth(oracle):
    """Deep residual stream (256 layers, hidden 1024, 64 tokens, P = 8): with
    both roundings fed back the error against the exact sum stays at the level
    of one call instead of growing with depth [rit.work "Echo 4-bit GPU
    communication", section "How Echo returns the error to later calls":
    with compensation the partial sum of the error stays bounded and does not
    grow with depth]. Every layer is compared bit for bit with the oracle."""
    import torch
    torch.backends.cuda.matmul.allow_tf32 = False
    P, hidden, tokens, layers, seed = 8, 1024, 64, 256, 0
    n = hidden * tokens
    x0 = torch.from_numpy(wl.residual_init(tokens, hidden, seed)).cuda()

    def partials(x, layer):
        xn = x / torch.sqrt(torch.mean(x.double() ** 2, dim=1, keepdim=True)).float()
        return torch.stack([(xn @ wl.residual_weight(layer, r, hidden, seed, device=x.device))
                            / float(np.sqrt(hidden * P)) for r in range(P)])

    runs = {"default": FullCompare(oracle, P, n, "fp32"),
            "both": FullCompare(oracle, P, n, "fp32", variant=OWNER_SUM | SENDER_EF)}
    x = {k: x0.clone() for k in list(runs) + ["ex"]}
    rel = {k: {} for k in runs}
    try:
        for layer in range(layers):
            pe = partials(x["ex"], layer)
            x["ex"] = (x["ex"].double() + pe.double().sum(0)).float()
            for key, fc in runs.items():
                ref = fc.call(partials(x[key], layer).reshape(P, n).cpu().numpy())
                x[key] = x[key] + torch.from_numpy(ref["out"]).cuda().reshape(tokens, hidden)
            if layer + 1 in (16, 256):
                ne = float(torch.linalg.norm(x["ex"]))
                for key in runs:
                    rel[key][layer + 1] = float(torch.linalg.norm(x[key] - x["ex"])) / ne
    finally:
        for fc in runs.values():
            fc.close()
    assert rel["both"][256] < 1.3 * rel["both"][16], rel     # flat with depth
    assert rel["both"][256] < 0.7 * rel["default"][256], rel


@pytest.mark.parametrize("variant", VARIANTS, ids=VIDS)
def test_variant_host_end_to_end(oracle, variant):
    """Host buffers in, host result out, over several pipelined pieces: the
    sender errors and the state follow the pieces."""
    import torch
    from bit_error_compensated_rank_b200 import echo
    P, n = 4, 4 * 32 * 80000  # 10.24 M elements per rank: three pieces
    h = echo.Echo(P, n)
    h.set_variant(variant)
    try:
        f = np.zeros(n, np.float32)
        s = np.zeros(n, np.float32)
        eps = np.zeros((P, n), np.float32)
        for k in range(2):
            x = gaussian(P, n, seed=17, call=k)
            host_in = [torch.from_numpy(x[r].view(np.int16)).view(torch.bfloat16).pin_memory()
                       for r in range(P)]
            host_out = torch.empty(n, dtype=torch.bfloat16).pin_memory()
            h.allreduce_host(host_in, host_out)
            ref = oracle.allreduce(x, f, s, Params(), variant=variant, eps=eps)
            assert_same_bits(host_out.view(torch.int16).numpy().view(np.uint16), ref["out"], "host result")
            gf, gs = h.get_state(0)
            assert_same_bits(gf, f, "fast estimate")
            assert_same_bits(gs, s, "slow estimate")
            if variant & SENDER_EF:
                for r in range(P):
                    assert_same_bits(h.get_sender_state(0, r), eps[r], f"sender error rank {r}")
    finally:
        h.close()
