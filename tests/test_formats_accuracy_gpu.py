"""Accuracy against wire bytes for the scale formats and group sizes, on the
inference-shaped and the deep-residual workloads.

Parity of every format with the oracle is tested elsewhere; here the CUDA
path alone runs each format and the results are compared with exact sums:

* Qwen3-8B-shaped inference (P = 4, 2048 tokens x 4096 hidden bf16, 72
  calls, channel-scaled partials with 1 % outlier channels, forward state):
  the mean relative error of one call, |Y - S| / |S|, and the relative size
  of the running total of injected error after all calls,
  |sum_k (Y_k - S_k)| / |S_1|;
* deep residual stream (256 layers, hidden 1024, 64 tokens, binary32, P = 8):
  |x - x_exact| / |x_exact| after 16, 64 and 256 layers.

Smaller groups and binary16 scales follow each group's maximum more closely
and cost more wire bytes [rit.work "Echo 4-bit GPU communication": the 4-bit
format trades volume against accuracy]. The test asserts that ordering and
prints one table row per format.
"""
import json

import numpy as np
import pytest

from bit_error_compensated_rank_b200 import workloads as wl

pytestmark = pytest.mark.gpu

# (name, group, variant bits)
FORMATS = [("pow2-g16", 16, 0), ("pow2-g32", 32, 0), ("pow2-g64", 64, 0), ("pow2-g128", 128, 0),
           ("fp16-g32", 32, 4), ("fp16-g128", 128, 4)]


def _wire_bytes(group, variant):
    return 0.5 + (2 if variant & 4 else 1) / group


def _inference(group, variant):
    import torch
    from bit_error_compensated_rank_b200 import echo
    P, tokens, hidden, calls = 4, 2048, 4096, 72
    n = tokens * hidden
    sigma = torch.from_numpy(wl.channel_scale(hidden, seed=0)).cuda()
    h = echo.Echo(P, n, echo.ECHO_BF16, group)
    if variant:
        h.set_variant(variant)
    send = [torch.empty(n, device="cuda", dtype=torch.bfloat16) for _ in range(P)]
    recv = [torch.empty_like(t) for t in send]
    total = torch.zeros(n, device="cuda", dtype=torch.float64)
    rel = []
    first = None
    try:
        for k in range(calls):
            for r in range(P):
                wl.torch_channel_scaled_(send[r], sigma, seed=0, call=k, rank=r)
            S = torch.stack([t.double() for t in send]).sum(0)
            h.allreduce_out(send, recv, 0)
            Y = recv[0].double()
            rel.append(float(torch.linalg.norm(Y - S) / torch.linalg.norm(S)))
            total += Y - S
            if first is None:
                first = float(torch.linalg.norm(S))
    finally:
        h.close()
    return {"call_rel": float(np.mean(rel)), "total_rel": float(torch.linalg.norm(total)) / first}


def _residual(group, variant):
    import torch
    from bit_error_compensated_rank_b200 import echo
    torch.backends.cuda.matmul.allow_tf32 = False
    P, hidden, tokens, layers, seed = 8, 1024, 64, 256, 0
    n = hidden * tokens
    x = torch.from_numpy(wl.residual_init(tokens, hidden, seed)).cuda()
    xe = x.clone()
    h = echo.Echo(P, n, echo.ECHO_FP32, group)
    if variant:
        h.set_variant(variant)
    scale = 1.0 / float(np.sqrt(hidden * P))
    out = {}
    try:
        for layer in range(layers):
            ws = [wl.residual_weight(layer, r, hidden, seed, device=x.device) for r in range(P)]

            def parts(v):
                vn = v / torch.sqrt(torch.mean(v.double() ** 2, dim=1, keepdim=True)).float()
                return [((vn @ w) * scale).reshape(-1).contiguous() for w in ws]

            pe = parts(xe)
            xe = (xe.double() + torch.stack(pe).double().sum(0).reshape(tokens, hidden)).float()
            bufs = parts(x)
            h.allreduce(bufs, 0)
            x = x + bufs[0].reshape(tokens, hidden)
            if layer + 1 in (16, 64, 256):
                out[f"rel_{layer + 1}"] = float(torch.linalg.norm(x - xe) / torch.linalg.norm(xe))
    finally:
        h.close()
    return out


def test_formats_accuracy_vs_bytes():
    rows = {}
    for name, group, variant in FORMATS:
        row = {"bytes_per_elem": _wire_bytes(group, variant)}
        row.update(_inference(group, variant))
        row.update(_residual(group, variant))
        rows[name] = row
        print(json.dumps({"format": name, **{k: round(v, 6) for k, v in row.items()}}), flush=True)
    # finer groups: smaller per-call error
    c = [rows[f"pow2-g{g}"]["call_rel"] for g in (16, 32, 64, 128)]
    assert c[0] < c[1] < c[2] < c[3], c
    # binary16 scales beat power-of-two scales at the same group size
    for g in (32, 128):
        assert rows[f"fp16-g{g}"]["call_rel"] < rows[f"pow2-g{g}"]["call_rel"], rows
    # the compensated residual stream stays near the exact one for every format
    for name, row in rows.items():
        assert row["rel_256"] < 0.5, (name, row)
