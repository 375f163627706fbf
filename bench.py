"""Benchmark of the Echo error-compensated 4-bit all-reduce on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl echo|reference]
                    [--mode simulated|sharded|replicas] [--config 1|2|4|5] [--sweep]

Workload (one step = one all-reduce call, the whole hot path: compensate +
quantise + pack, owner reduce + requantise, gather + dequantise): P = 8
simulated tensor-parallel ranks, a 1 GiB bf16 message per rank (2^29
elements), partials N(0, 1) with 0.1 % of values at 50x, group 32,
compensation on, forward state. The ranks are 8 buffers in one GPU's HBM.

Metric: bf16-equivalent all-reduce bandwidth, algbw = 2 n / t_call (the
nccl-tests definition), and the call's fraction of the HBM roofline, where
the roofline time is the three kernels' algorithmic bytes divided by the
measured HBM copy bandwidth.

Modes (``--mode``; the default is ``simulated`` at N = 1, ``sharded`` at
N > 1):

* ``simulated``: one handle, the P ranks are P buffers in one GPU's HBM.
* ``sharded``: the same P-rank all-reduce with one handle per rank
  (echo_dist_*), the P ranks spread over the N processes (P/N each, one
  process per GPU), the wire stored straight into the other ranks' blocks
  (peer stores over NVLink between GPUs) and the stages ordered by events.
  The problem is fixed as N grows (strong scaling) and the value is the
  all-reduce's algbw; at N = 8 it is the P = 8, 1 GiB all-reduce over NVLink.
* ``replicas``: every GPU runs its own independent P-rank simulated problem
  (weak scaling, nothing crosses GPUs); the value is the sum of all GPUs'
  work divided by the slowest GPU's time.

``--config 1|2|4|5`` prints one line for another of the five workloads
(per-call time issued one by one and replayed from a CUDA graph, algbw,
roofline fraction; for the deep residual stream also the distance to the
exact sum by depth) instead of the benchmark line.

``--impl reference`` times the plain CPU oracle instead (the slow reference
program this library is checked against), on a bounded sample of the same
workload per step; under torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "bf16-equiv all-reduce GB/s and % of HBM roofline at P=8, 1 GiB msg"
UNIT = "GB/s"
P = 8
N_ELEMS = 1 << 29          # 1 GiB of bf16 per rank
SEED = 0
WORKLOAD = "echo int4 all-reduce, P=8 ranks x 1 GiB bf16 per rank (2^29 elements), group 32, " \
           "compensation on, fwd state, partials N(0,1) with 0.1% at 50x"
HBM_FALLBACK_GBS = 6650.0  # used only when MEASURED_PEAKS.json is absent
L2_BYTES = 126 * 10 ** 6
# where the rounding errors are fed back, and the scale format (see
# include/echo.h, echo_set_variant)
VARIANTS = {"default": 0, "owner_sum": 1, "sender_ef": 2, "both": 3, "fp16_scale": 4}
# CPU baseline / reference arm samples (elements per rank, same distribution)
CPU_SAMPLE_N = 1 << 20
REF_SAMPLE_N = 1 << 18


# ---------------------------------------------------------------------------
# process group plumbing
# ---------------------------------------------------------------------------
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(world: int, backend: str):
    import datetime
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(value: float, world: int, device=None) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, world: int, device=None) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------------------
# measured peaks and clocks
# ---------------------------------------------------------------------------
def hbm_peak() -> tuple[float, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            return float(json.load(fh)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return HBM_FALLBACK_GBS, "fallback"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str, period_ms: int = 50):
        self.gpu_id = gpu_id
        self.period_ms = period_ms
        self.rows: list[list[str]] = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(self.period_ms)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([c.strip() for c in line.split(",")])

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for row in self.rows:
            if len(row) < 8:
                continue
            try:
                sm.append(float(row[0]))
                smax.append(float(row[1]))
            except ValueError:
                continue
            for name, val in zip(names, row[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def gpu_selector(local_rank: int) -> str:
    import torch
    try:
        uuid = str(torch.cuda.get_device_properties(local_rank).uuid)
        return uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            return vis.split(",")[local_rank]
        return str(local_rank)


# ---------------------------------------------------------------------------
# the CPU oracle (baseline leg and reference arm)
# ---------------------------------------------------------------------------
def oracle_sample_rate(n_sample: int, budget_s: float, min_calls: int, max_calls: int, seed: int,
                       variant: int = 0):
    """Time the oracle on P x n_sample bf16 partials of the workload's
    distribution, call after call (state carried), until budget_s is spent."""
    import numpy as np
    from bit_error_compensated_rank_b200 import workloads as wl
    from oracle.oracle import Oracle, Params
    orc = Oracle()
    f = np.zeros(n_sample, np.float32)
    s = np.zeros(n_sample, np.float32)
    eps = np.zeros((P, n_sample), np.float32)
    times = []
    t_all = time.perf_counter()
    k = 0
    while k < min_calls or (time.perf_counter() - t_all < budget_s and k < max_calls):
        x = wl.outlier_gaussian(P, n_sample, seed=seed, call=k)
        t0 = time.perf_counter()
        orc.allreduce(x, f, s, Params(), want_wire=False, variant=variant, eps=eps)
        times.append(time.perf_counter() - t0)
        k += 1
    return times


def host_info() -> dict:
    """CPU model, logical cores and RAM of the host the oracle runs on."""
    info = {"nproc": os.cpu_count(), "cpu_model": None, "ram_gb": None}
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    info["cpu_model"] = line.split(":", 1)[1].strip()
                    break
        with open("/proc/meminfo") as fh:
            for line in fh:
                if line.startswith("MemTotal"):
                    info["ram_gb"] = round(int(line.split()[1]) / 2 ** 20, 1)
                    break
    except OSError:
        pass
    return info


class one_core:
    """Pin this process to one core (the first it may use) while timing the
    single-threaded oracle; restore the previous set afterwards."""

    def __enter__(self):
        self.prev = None
        if hasattr(os, "sched_getaffinity"):
            try:
                self.prev = os.sched_getaffinity(0)
                os.sched_setaffinity(0, {min(self.prev)})
            except OSError:
                self.prev = None
        return self

    def __exit__(self, *exc):
        if self.prev is not None:
            try:
                os.sched_setaffinity(0, self.prev)
            except OSError:
                pass
        return False


def cpu_baseline_leg(variant: int = 0) -> dict:
    with one_core():
        times = oracle_sample_rate(CPU_SAMPLE_N, budget_s=15.0, min_calls=3, max_calls=80, seed=1,
                                   variant=variant)
    t = sum(times) / len(times)
    return {
        "value": round(2 * CPU_SAMPLE_N / t / 1e9, 6), "unit": UNIT, "cores": 1, "kind": "oracle",
        "sample": f"P={P} x 2^20 bf16 elements per rank (2 MiB), same distribution, compensation on, "
                  f"{len(times)} sequential calls, {sum(times):.1f} s single-threaded on one pinned "
                  f"core; value = 2*n/t per call (bf16-equivalent)",
        "host": host_info(),
    }


def run_reference(args, rank: int, world: int) -> dict | None:
    if rank != 0:
        return None
    with one_core():
        times = oracle_sample_rate(REF_SAMPLE_N, budget_s=0.0, min_calls=args.warmup + args.steps,
                                   max_calls=args.warmup + args.steps, seed=2)
    timed = times[args.warmup:]
    t = sum(timed) / len(timed)
    value = 2 * REF_SAMPLE_N / t / 1e9
    sample = (f"P={P} x 2^18 bf16 elements per rank per step (512 KiB), same distribution as the "
              f"1 GiB workload, compensation on; oracle single-threaded on the host")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(t * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD, "P": P, "n_per_rank": N_ELEMS, "sample_n_per_rank": REF_SAMPLE_N,
                   "element_dtype": "bf16", "wire": "int4 codes + scales",
                   "parallelism": f"{world} independent replica(s)"},
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": sample, "host": host_info()},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------
# DRAM traffic per element of n for each kernel from one ncu capture
# ((dram__bytes_read.sum + dram__bytes_write.sum) / n, captured at P = 8,
# n = 2^26 and scaled by n, since the traffic grows in proportion); reported
# only while the kernel source still has the hash it had when captured.
NCU_TRAFFIC = {
    "k1_compensate_quantize_pack": {"bytes_per_elem": 28.059, "source_sha": "0929b049589af0b2"},
}


def workload_name(args) -> str:
    name = WORKLOAD if args.group == 32 else WORKLOAD.replace("group 32", f"group {args.group}")
    if P != 8:
        name = name.replace("P=8 ranks", f"P={P} ranks")
    return name if args.variant == "default" else f"{name}, variant {args.variant}"


def _source_hash(path: str) -> str:
    """First 16 hex digits of the sha256 of a kernel's .cu file followed by
    its .cuh body, when it has one."""
    import hashlib
    h = hashlib.sha256()
    for p in (path, path[:-3] + ".cuh"):
        if os.path.exists(p):
            with open(p, "rb") as fh:
                h.update(fh.read())
    return h.hexdigest()[:16]


def run_echo(args, rank: int, world: int, local: int) -> dict | None:
    import torch
    from bit_error_compensated_rank_b200 import echo
    from bit_error_compensated_rank_b200 import workloads as wl

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    # whole groups on every rank: round down to a multiple of P * max(group, 32)
    n = args.n - args.n % (P * max(args.group, 32))
    stream = torch.cuda.current_stream(device)

    # inputs resident in HBM before timing; outputs to separate buffers so
    # every step sees the same fresh partials (out-of-place call, same bytes)
    send = [torch.empty(n, dtype=torch.bfloat16, device=device) for _ in range(P)]
    recv = [torch.empty(n, dtype=torch.bfloat16, device=device) for _ in range(P)]
    for r in range(P):
        wl.torch_outlier_gaussian_(send[r], seed=SEED + 1000 * rank, call=0, rank=r)
    variant = VARIANTS[args.variant]
    h = echo.Echo(P, n, echo.ECHO_BF16, args.group)
    if variant:
        h.set_variant(variant)
    # the three pipelined kernels at any --n, unless --fused-limit lets this
    # size run as one kernel
    h.set_fused_limit(0 if args.fused_limit is None else args.fused_limit)
    fused = call_path(h, n) == "one kernel"
    mb = echo.echo_model_bytes_ex(P, n, args.group, echo.ECHO_BF16, True, variant)
    torch.cuda.synchronize()

    for _ in range(args.warmup):
        h.allreduce_out(send, recv, echo.ECHO_FWD, stream)
    torch.cuda.synchronize()

    clocks = ClockSampler(gpu_selector(local))
    clocks.start()
    h.set_timing(True)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    barrier(world, device)
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(args.steps):
        h.allreduce_out(send, recv, echo.ECHO_FWD, stream)
    end.record(stream)
    torch.cuda.synchronize()
    barrier(world, device)
    clk = clocks.stop()
    h.set_timing(False)
    kern_ms, timed_calls = h.kernel_ms_total()
    elapsed_ms = start.elapsed_time(end)
    ms_step = max_over_ranks(elapsed_ms / args.steps, world, device)
    assert timed_calls == args.steps

    # whole-job throughput: every GPU moved 2n bf16-equivalent bytes per step
    total_bytes = sum_over_ranks(2.0 * n * args.steps, world, device)
    value = total_bytes / (ms_step * args.steps * 1e-3) / 1e9
    peak, peak_kind = hbm_peak()
    call_bytes = mb["total"]
    call_frac = call_bytes / (ms_step * 1e-3) / (peak * 1e9)
    # On one GPU the P simulated ranks share one requantised buffer, which
    # kernel 3 reads once instead of once per rank: (P-1) wire reads fewer
    # than the P-GPU model above, whose fraction can therefore pass 1.
    min_bytes = call_bytes - mb["link"] // 2

    k_avg = [t / timed_calls for t in kern_ms]
    names = ["k1_compensate_quantize_pack", "k2_owner_reduce_requant", "k3_gather_dequant"]
    k_bytes = [mb["k1"], mb["k2"], mb["k3"]]
    if fused:  # one kernel, timed as kernel 1, with its own bytes
        names, k_avg, k_bytes = ["kf_fused_allreduce"], k_avg[:1], [fused_bytes(P, n, 2, args.group, True, variant)]
        call_bytes = k_bytes[0]
        call_frac = call_bytes / (ms_step * 1e-3) / (peak * 1e9)
        min_bytes = call_bytes
    dom = max(range(len(names)), key=lambda i: k_bytes[i])
    achieved = k_bytes[dom] / (k_avg[dom] * 1e-3) / 1e9
    src = os.path.join(ROOT, "bit_error_compensated_rank_b200", "csrc", names[dom] + ".cu")
    traffic = None
    # captured for the default variant and group
    rec = NCU_TRAFFIC.get(names[dom]) if variant == 0 and args.group == 32 and P == 8 else None
    if rec and rec["source_sha"] == _source_hash(src):
        traffic = round(rec["bytes_per_elem"] * n)

    # end to end: pinned host partials in, host result out, through the C ABI
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(h, send, n, args, device, world)

    result = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        # arithmetic in binary32 (restores, sums, estimates) on bf16 partials and
        # outputs with 4-bit codes on the wire
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": workload_name(args),
                   "variant": args.variant, "P": P, "n_per_rank": n, "group": args.group,
                   "element_dtype": "bf16", "wire": "int4 codes + scales",
                   "mode": "simulated" if world == 1 else "replicas",
                   "parallelism": f"{world} independent replica(s), ranks simulated in HBM",
                   "l2": "inputs larger than L2 (8 GiB of partials per GPU vs 126 MB L2)"},
        "hbm_roofline_frac": round(call_frac, 4),
        "hbm_roofline": {"model_bytes_per_call": call_bytes,
                         "bytes_per_elem": round(call_bytes / n, 5),
                         "peak_gbs": peak, "peak_kind": peak_kind,
                         "ideal_ms": round(call_bytes / (peak * 1e9) * 1e3, 4),
                         "model": "one kernel: partials and state read, both wires, state and outputs written"
                                  if fused else "P-GPU: every rank reads its own copy of the requantised wire"},
        "path": "one kernel" if fused else "three kernels",
        "single_gpu_min_bytes_per_elem": round(min_bytes / n, 5),
        "single_gpu_min_frac": round(min_bytes / (ms_step * 1e-3) / (peak * 1e9), 4),
        "busbw": round(value * 2 * (P - 1) / P, 3),
        "kernel_ms": {names[i]: round(k_avg[i], 4) for i in range(len(names))},
        "kernel_frac": {names[i]: round(k_bytes[i] / (k_avg[i] * 1e-3) / 1e9 / peak, 4)
                        for i in range(len(names))},
        "link_bytes_per_call": mb["link"],
        "roofline": {"kernel": names[dom], "bound": "hbm", "achieved": round(achieved, 1),
                     "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": traffic, "peak_kind": peak_kind},
        "gpu_launches": (1 if fused else 3) * args.steps,
        "clocks": clk,
    }
    if e2e is not None:
        result["e2e"] = e2e
    h.close()
    return result if rank == 0 else None


# Peer copy bandwidth per direction per GPU measured on this machine's B200s over
# NVLink 5 (the denominator of the sharded mode's link fraction; nominal 900).
NVLINK_PEER_GBS = 770.0


def shard_ranks(P: int, world: int, rank: int) -> list[int]:
    """The all-reduce ranks that process ``rank`` of ``world`` holds: P/world
    consecutive ranks."""
    if P % world:
        raise ValueError(f"{P} ranks do not split evenly over {world} processes")
    per = P // world
    return list(range(rank * per, (rank + 1) * per))


def cross_gpu_link_bytes(P: int, n_gpus: int, link_bytes: int) -> int:
    """Wire bytes one GPU sends to the other GPUs per call when the P ranks
    are spread L = P/N per GPU. ``link_bytes`` is the P-GPU figure 2(P-1)*W,
    W the wire bytes of a whole message, so a segment's wire is W/P. Each of a
    GPU's L ranks sends its segments for the P - L owners on other GPUs, and
    each of its L owners sends its requantised segment to those P - L ranks:
    2 L (P - L) W / P, which is 2(P-1)/P * W at one rank per GPU."""
    if n_gpus <= 1:
        return 0
    L = P // n_gpus
    W = link_bytes // (2 * (P - 1))
    return 2 * L * (P - L) * W // P


def run_sharded(args, rank: int, world: int, local: int) -> dict | None:
    """The P-rank all-reduce with one handle per rank (echo_dist_*), the
    ranks spread over the processes (P/world each); strong scaling."""
    import torch
    from bit_error_compensated_rank_b200 import echo
    from bit_error_compensated_rank_b200 import workloads as wl

    dev_index = 0 if args.one_gpu else local
    torch.cuda.set_device(dev_index)
    device = torch.device("cuda", dev_index)
    dist = init_dist(world, "gloo")  # host barriers and the handle exchange only: no data
    mine = shard_ranks(P, world, rank)
    n = args.n - args.n % (P * max(args.group, 32))
    stream = torch.cuda.current_stream(device)
    xs = [torch.empty(n, dtype=torch.bfloat16, device=device) for _ in mine]
    outs = [torch.empty(n, dtype=torch.bfloat16, device=device) for _ in mine]
    for x, r in zip(xs, mine):
        wl.torch_outlier_gaussian_(x, seed=SEED, call=0, rank=r)
    variant = VARIANTS[args.variant]
    ds = [echo.DistEcho(P, r, n, echo.ECHO_BF16, args.group) for r in mine]
    for d in ds:
        if variant:
            d.set_variant(variant)
    blobs = [d.export() for d in ds]
    if world > 1:
        gathered = [None] * world
        dist.all_gather_object(gathered, blobs)
        blobs = [b for part in gathered for b in part]
    for d in ds:
        d.connect(blobs)

    def bar():
        barrier(world)

    def call():
        echo.dist_allreduce(ds, xs, outs, bar, echo.ECHO_FWD, stream, sync=args.host_ordered)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    bar()
    clocks = ClockSampler(gpu_selector(dev_index))
    clocks.start()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    bar()
    start.record(stream)
    for _ in range(args.steps):
        call()
    end.record(stream)
    torch.cuda.synchronize()
    bar()
    clk = clocks.stop()
    ms_step = max_over_ranks(start.elapsed_time(end) / args.steps, world)
    stage_ms = sharded_stage_ms(ds, xs, outs, bar, stream, args)

    mb = echo.echo_model_bytes_ex(P, n, args.group, echo.ECHO_BF16, True, variant)
    n_gpus = 1 if args.one_gpu else world
    peak, peak_kind = hbm_peak()
    gpu_bytes = mb["total"] * len(mine) // P  # the model is the same for every rank
    hbm_achieved = gpu_bytes / (ms_step * 1e-3) / 1e9
    link = cross_gpu_link_bytes(P, n_gpus, mb["link"])
    value = 2.0 * n / (ms_step * 1e-3) / 1e9

    e2e = None
    if not args.no_e2e:
        e2e = run_sharded_e2e(ds, xs, outs, n, args, device, world, bar)
    result = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": n_gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": workload_name(args), "mode": "sharded", "variant": args.variant, "P": P,
                   "n_per_rank": n, "group": args.group, "element_dtype": "bf16",
                   "wire": "int4 codes + scales",
                   "parallelism": f"{P} ranks as one handle each, {len(mine)} per process, {world} "
                                  f"process(es) on {n_gpus} GPU(s); wire stored into the other ranks' "
                                  f"blocks, stages ordered by "
                                  f"{'host synchronisation' if args.host_ordered else 'events'}",
                   "l2": "inputs larger than L2" if P // n_gpus * n * 2 > L2_BYTES else "inputs fit in L2"},
        "busbw": round(value * 2 * (P - 1) / P, 3),
        "hbm_roofline_frac": round(hbm_achieved / peak, 4),
        "roofline": {"kernel": "whole call (three stages)", "bound": "hbm", "achieved": round(hbm_achieved, 1),
                     "peak": peak, "unit": "GB/s", "frac": round(hbm_achieved / peak, 4), "traffic": None,
                     "peak_kind": peak_kind, "bytes_per_gpu_per_call": gpu_bytes},
        "link_bytes_per_gpu_per_call": link,
        # after the timed region: each stage of this process's ranks, the
        # waits on the other ranks' events included (rank 0's process)
        "stage_ms": stage_ms,
        "gpu_launches": 3 * len(mine) * args.steps,
        "clocks": clk,
    }
    if link:
        result["link"] = {"achieved_gbs": round(link / (ms_step * 1e-3) / 1e9, 1),
                          "peak_gbs": NVLINK_PEER_GBS, "peak_kind": "measured peer copy per direction",
                          "frac": round(link / (ms_step * 1e-3) / 1e9 / NVLINK_PEER_GBS, 4)}
    if e2e is not None:
        result["e2e"] = e2e
    torch.cuda.synchronize()
    bar()
    for d in ds:
        d.close()
    return result if rank == 0 else None


def sharded_stage_ms(ds, xs, outs, bar, stream, args) -> list[float]:
    """Mean time of each of the three stages over ``args.steps`` more calls,
    from CUDA events recorded between the stages on the launching stream."""
    import torch
    from bit_error_compensated_rank_b200 import echo
    calls = []
    for _ in range(args.steps):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        ev[0].record(stream)
        for k in (1, 2, 3):
            for d, x, out in zip(ds, xs, outs):
                d.stage(k, x, out, echo.ECHO_FWD, stream)
            ev[k].record(stream)
            if k < 3:
                bar()
        calls.append(ev)
    torch.cuda.synchronize()
    bar()
    return [round(statistics.mean(ev[k - 1].elapsed_time(ev[k]) for ev in calls), 4) for k in (1, 2, 3)]


def run_sharded_e2e(ds, xs, outs, n, args, device, world, bar) -> dict:
    """Per step: every local rank's partial from pinned host memory to the
    device, the all-reduce, and the result back to pinned host memory."""
    import torch
    from bit_error_compensated_rank_b200 import echo
    steps = max(1, min(args.steps, args.e2e_steps))
    try:
        host_in = [torch.empty(n, dtype=torch.bfloat16, pin_memory=True) for _ in xs]
        host_out = torch.empty(n, dtype=torch.bfloat16, pin_memory=True)
    except RuntimeError as exc:
        return {"value": None, "unit": UNIT, "error": f"pinned host allocation failed: {exc}"}
    for h, x in zip(host_in, xs):
        h.copy_(x)
    stream = torch.cuda.current_stream(device)

    def step():
        for x, h in zip(xs, host_in):
            x.copy_(h, non_blocking=True)
        echo.dist_allreduce(ds, xs, outs, bar, echo.ECHO_FWD, stream, sync=args.host_ordered)
        host_out.copy_(outs[0], non_blocking=True)

    step()
    torch.cuda.synchronize()
    bar()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        step()
    end.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(start.elapsed_time(end) / steps, world)
    return {"value": round(2.0 * n / (ms * 1e-3) / 1e9, 3), "unit": UNIT,
            "h2d_bytes_per_step": int(sum_over_ranks(2.0 * n * len(xs), world)),
            "d2h_bytes_per_step": int(sum_over_ranks(2.0 * n, world)),
            "ms_per_step": round(ms, 3), "steps": steps}


# The other four workloads: shape and inputs (the headline is the third).
CONFIG_DESC = {
    1: "P=2, one 4096-element bf16 partial per rank (1 token x hidden 4096), N(0,1), group 32, "
       "8 calls, compensation on, seed 0",
    2: "Qwen3-8B-shaped inference: P=4, 2048 tokens x 4096 hidden bf16, 72 calls, channel-scaled "
       "partials (sigma_c log-uniform [0.1,1], 1% channels x20), forward state only",
    4: "Llama-3-8B-shaped training step: P=4, 2 x 4096 tokens x 4096 hidden bf16, 64 forward calls "
       "(channel-scaled) then 64 backward calls (1e-3 Student-t nu=3), separate state",
    5: "deep residual stream: P=8, 64 tokens x hidden 1024 binary32, 256 layers, pre-norm partials "
       "(x/rms(x)) W_r / sqrt(1024 P); compensation on vs off vs sender feedback vs exact sum",
}


def time_sequence(h, seq, outs, stream, min_ms: float = 60.0) -> tuple[float, float, int]:
    """Per-call time of a sequence of out-of-place calls ``seq`` = [(inputs,
    phase), ...] on handle ``h``: (a) issued one by one from Python, and (b)
    captured once in a CUDA graph and replayed (the GPU time). Returns
    (eager ms, graph ms, repetitions of the sequence)."""
    import torch

    def run_once(st):
        for xs, phase in seq:
            h.allreduce_out(xs, outs, phase, st)

    run_once(stream)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    run_once(stream)
    end.record(stream)
    torch.cuda.synchronize()
    reps = max(2, min(2000, int(min_ms / max(start.elapsed_time(end), 1e-3)) + 1))
    start.record(stream)
    for _ in range(reps):
        run_once(stream)
    end.record(stream)
    torch.cuda.synchronize()
    eager = start.elapsed_time(end) / (reps * len(seq))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run_once(None)
    graph.replay()
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(reps):
        graph.replay()
    end.record(stream)
    torch.cuda.synchronize()
    replayed = start.elapsed_time(end) / (reps * len(seq))
    del graph
    return eager, replayed, reps


def residual_partials(x, layer: int, P: int, hidden: int, seed: int):
    """Pre-norm tensor-parallel partials of one layer of the deep residual
    stream: (x / rms(x)) W_{layer,r} / sqrt(hidden * P), r = 0..P-1."""
    import torch
    from bit_error_compensated_rank_b200 import workloads as wl
    xn = x / torch.sqrt(torch.mean(x.double() ** 2, dim=1, keepdim=True)).float()
    scale = 1.0 / math.sqrt(hidden * P)
    return [(xn @ wl.residual_weight(layer, r, hidden, seed, device=x.device)) * scale for r in range(P)]


def residual_errors(P: int, tokens: int, hidden: int, layers: int, seed: int) -> dict:
    """The deep residual stream run three ways through the CUDA path
    (compensation on, off, and on with sender feedback) beside the exact sum
    of the partials (binary64), from the same start: |x - x_exact| / |x_exact|
    and |x - x_exact| per layer, reported at layers 1, 2, 4, ..., ``layers``."""
    import torch
    from bit_error_compensated_rank_b200 import echo
    from bit_error_compensated_rank_b200 import workloads as wl
    torch.backends.cuda.matmul.allow_tf32 = False
    n = tokens * hidden
    x0 = torch.from_numpy(wl.residual_init(tokens, hidden, seed)).cuda()
    runs = {"on": (True, 0), "off": (False, 0), "sender_ef": (True, echo.ECHO_VARIANT_SENDER_EF)}
    handles = {}
    for key, (enable, variant) in runs.items():
        h = echo.Echo(P, n, echo.ECHO_FP32)
        h.set_params(enable=enable)
        if variant:
            h.set_variant(variant)
        handles[key] = h
    x = {k: x0.clone() for k in list(runs) + ["exact"]}
    marks = [2 ** k for k in range(int(math.log2(layers)) + 1)]
    out = {"layers": marks, "rel": {k: [] for k in runs}, "abs": {k: [] for k in runs}}
    for layer in range(layers):
        pe = residual_partials(x["exact"], layer, P, hidden, seed)
        x["exact"] = (x["exact"].double() + torch.stack(pe).double().sum(0)).float()
        for key, h in handles.items():
            parts = [t.reshape(-1).contiguous() for t in residual_partials(x[key], layer, P, hidden, seed)]
            h.allreduce(parts, 0)
            x[key] = x[key] + parts[0].reshape(tokens, hidden)
        if layer + 1 in marks:
            ref = float(torch.linalg.norm(x["exact"].double()))
            for key in runs:
                d = float(torch.linalg.norm((x[key] - x["exact"]).double()))
                out["abs"][key].append(round(d, 6))
                out["rel"][key].append(round(d / ref, 6))
    for h in handles.values():
        h.close()
    return out


def fused_bytes(Pc: int, n: int, ebytes: int, group: int = 32, enable: bool = True, variant: int = 0) -> int:
    """Algorithmic HBM bytes of one call run as one kernel: the P partials and
    the state read; both wires, the state and the P outputs written; sender
    feedback's errors read and written. Nothing is read back."""
    wire = n // 2 + n // group * (2 if variant & 4 else 1)
    b = Pc * ebytes * n + (Pc + 1) * wire + Pc * ebytes * n
    if enable:
        b += 16 * n
    if variant & 2:
        b += 8 * Pc * n
    return b


def call_path(h, n: int) -> str:
    return "one kernel" if n <= h.fused_limit() else "three kernels"


def run_config(args) -> dict:
    """One line for workload ``args.config`` (1, 2, 4 or 5)."""
    import numpy as np
    import torch
    from bit_error_compensated_rank_b200 import echo
    from bit_error_compensated_rank_b200 import workloads as wl

    torch.cuda.set_device(0)
    stream = torch.cuda.current_stream()
    peak, peak_kind = hbm_peak()
    cfg = args.config
    if cfg == 1:
        Pc, n, code = 2, 4096, echo.ECHO_BF16
        seq_inputs = []
        for k in range(8):
            x = torch.from_numpy(wl.gaussian(Pc, n, seed=0, call=k).view(np.int16)).cuda()
            seq_inputs.append(([x[r].view(torch.bfloat16) for r in range(Pc)], 0))
    elif cfg in (2, 4):
        Pc, hidden, code = 4, 4096, echo.ECHO_BF16
        tokens = 2048 if cfg == 2 else 2 * 4096
        n = tokens * hidden
        sigma = torch.from_numpy(wl.channel_scale(hidden, seed=0 if cfg == 2 else 1)).cuda()
        pool = 72 if cfg == 2 else 8  # distinct input sets (config 4 cycles 8 per phase)
        fwd = []
        for k in range(pool):
            bufs = [torch.empty(n, dtype=torch.bfloat16, device="cuda") for _ in range(Pc)]
            for r in range(Pc):
                wl.torch_channel_scaled_(bufs[r], sigma, seed=cfg, call=k, rank=r)
            fwd.append(bufs)
        if cfg == 2:
            seq_inputs = [(fwd[k], 0) for k in range(72)]
        else:
            bwd = []
            for k in range(pool):
                bufs = [torch.empty(n, dtype=torch.bfloat16, device="cuda") for _ in range(Pc)]
                for r in range(Pc):
                    wl.torch_student_t_(bufs[r], seed=cfg, call=k, rank=r)
                bwd.append(bufs)
            seq_inputs = [(fwd[k % pool], 0) for k in range(64)] + [(bwd[k % pool], 1) for k in range(64)]
    elif cfg == 5:
        Pc, hidden, tokens, code = 8, 1024, 64, echo.ECHO_FP32
        n = hidden * tokens
        x0 = torch.from_numpy(wl.residual_init(tokens, hidden, 0)).cuda()
        seq_inputs = [([t.reshape(-1).contiguous() for t in residual_partials(x0, layer, Pc, hidden, 0)], 0)
                      for layer in range(8)]
    else:
        raise ValueError(f"no workload {cfg}")
    ebytes = 2 if code == echo.ECHO_BF16 else 4
    outs = [torch.empty(n, dtype=torch.bfloat16 if code == echo.ECHO_BF16 else torch.float32, device="cuda")
            for _ in range(Pc)]
    h = echo.Echo(Pc, n, code)
    if args.fused_limit is not None:
        h.set_fused_limit(args.fused_limit)
    path = call_path(h, n)
    clocks = ClockSampler(gpu_selector(0))
    clocks.start()
    eager, graph, reps = time_sequence(h, seq_inputs, outs, stream)
    three = None
    if path == "one kernel":  # the three pipelined kernels on the same sequence, for comparison
        h.set_fused_limit(0)
        three = time_sequence(h, seq_inputs, outs, stream)
    clk = clocks.stop()
    h.close()
    mb = echo.echo_model_bytes(Pc, n, code, True)
    # the bytes of the path that ran: the one-kernel path reads no wire back
    path_bytes = fused_bytes(Pc, n, ebytes) if path == "one kernel" else mb["total"]
    frac_graph = path_bytes / (graph * 1e-3) / (peak * 1e9)
    line = {
        "config_line": cfg, "workload": CONFIG_DESC[cfg], "P": Pc, "n_per_rank": n,
        "element_dtype": "bf16" if code == echo.ECHO_BF16 else "fp32",
        "path": path,
        "calls_per_sequence": len(seq_inputs), "sequence_repetitions": reps,
        "us_per_call_eager": round(eager * 1e3, 2), "us_per_call_graph": round(graph * 1e3, 2),
        "algbw_GBs_eager": round(ebytes * n / (eager * 1e-3) / 1e9, 2),
        "algbw_GBs_graph": round(ebytes * n / (graph * 1e-3) / 1e9, 2),
        "bytes_per_call": path_bytes, "model_bytes_per_call_three_kernels": mb["total"],
        "roofline_frac_eager": round(path_bytes / (eager * 1e-3) / (peak * 1e9), 4),
        "roofline_frac_graph": round(frac_graph, 4), "peak_gbs": peak, "peak_kind": peak_kind,
        "l2_resident": mb["total"] < L2_BYTES,
        "regime": "launch-bound" if frac_graph < 0.5 else "hbm-bound",
        "link_bytes_per_call": mb["link"],
        "clocks": clk,
    }
    if three is not None:
        line["three_kernels"] = {"us_per_call_eager": round(three[0] * 1e3, 2),
                                 "us_per_call_graph": round(three[1] * 1e3, 2),
                                 "roofline_frac_graph": round(mb["total"] / (three[1] * 1e-3) / (peak * 1e9), 4)}
    if cfg == 4:
        line["inputs"] = "8 distinct input sets per phase, cycled over the 64 calls of each phase"
    if cfg == 5:
        line["inputs"] = "timing: 8 layers' partials from the start point, cycled"
        line["residual_error_vs_depth"] = residual_errors(Pc, tokens, hidden, 256, 0)
    return line


def run_e2e(h, send, n, args, device, world) -> dict:
    """Pinned host partials -> device -> all-reduce -> host result, per step."""
    import torch
    steps = max(1, min(args.steps, args.e2e_steps))
    try:
        host_in = [torch.empty(n, dtype=torch.bfloat16, pin_memory=True) for _ in range(P)]
        host_out = torch.empty(n, dtype=torch.bfloat16, pin_memory=True)
    except RuntimeError as exc:
        return {"value": None, "unit": UNIT, "error": f"pinned host allocation failed: {exc}"}
    for r in range(P):
        host_in[r].copy_(send[r])
    stream = torch.cuda.current_stream(device)
    h.allreduce_host(host_in, host_out, 0, stream)  # warm-up (allocates staging)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    barrier(world, device)
    start.record(stream)
    for _ in range(steps):
        h.allreduce_host(host_in, host_out, 0, stream)
    end.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(start.elapsed_time(end) / steps, world, device)
    total = sum_over_ranks(2.0 * n, world, device)
    return {"value": round(total / (ms * 1e-3) / 1e9, 3), "unit": UNIT,
            "h2d_bytes_per_step": P * n * 2, "d2h_bytes_per_step": n * 2,
            "ms_per_step": round(ms, 3), "steps": steps}


def run_sweep(args) -> None:
    """Message-size sweep (one JSON line per size, not the benchmark line):
    P = 8, bf16, n = 2^12 .. 2^sweep_max (default 2^29) elements per rank, CUDA-event time per call
    over enough calls to fill about 50 ms, inputs resident, out of place."""
    import torch
    from bit_error_compensated_rank_b200 import echo
    from bit_error_compensated_rank_b200 import workloads as wl
    torch.cuda.set_device(0)
    stream = torch.cuda.current_stream()
    peak, _ = hbm_peak()
    nmax = 1 << args.sweep_max
    send = [torch.empty(nmax, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    recv = [torch.empty(nmax, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    for r in range(P):
        wl.torch_outlier_gaussian_(send[r], seed=SEED, call=0, rank=r)
    variant = VARIANTS[args.variant]
    for k in range(12, args.sweep_max + 1):
        n = (1 << k) - (1 << k) % (P * max(args.group, 32))
        h = echo.Echo(P, n, echo.ECHO_BF16, args.group)
        if variant:
            h.set_variant(variant)
        if args.fused_limit is not None:
            h.set_fused_limit(args.fused_limit)
        path = call_path(h, n)
        s_views = [t[:n] for t in send]
        r_views = [t[:n] for t in recv]
        for _ in range(args.warmup):
            h.allreduce_out(s_views, r_views, 0, stream)
        torch.cuda.synchronize()
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        h.allreduce_out(s_views, r_views, 0, stream)
        end.record(stream)
        torch.cuda.synchronize()
        calls = max(5, min(2000, int(50.0 / max(start.elapsed_time(end), 1e-3))))
        # (a) calls issued one by one from Python: includes host submission
        start.record(stream)
        for _ in range(calls):
            h.allreduce_out(s_views, r_views, 0, stream)
        end.record(stream)
        torch.cuda.synchronize()
        ms = start.elapsed_time(end) / calls
        # (a') 16 calls timed one by one (events around each): the median
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(16)]
        for e_start, e_end in evs:
            e_start.record(stream)
            h.allreduce_out(s_views, r_views, 0, stream)
            e_end.record(stream)
        torch.cuda.synchronize()
        ms_median = statistics.median(a.elapsed_time(b) for a, b in evs)
        # (b) the same calls captured once in a CUDA graph and replayed: GPU time
        per_graph = min(calls, 50)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for _ in range(per_graph):
                h.allreduce_out(s_views, r_views, 0, None)
        graph.replay()
        torch.cuda.synchronize()
        reps = max(1, calls // per_graph)
        start.record(stream)
        for _ in range(reps):
            graph.replay()
        end.record(stream)
        torch.cuda.synchronize()
        ms_graph = start.elapsed_time(end) / (reps * per_graph)
        del graph
        mb = echo.echo_model_bytes_ex(P, n, args.group, echo.ECHO_BF16, True, variant)
        path_bytes = fused_bytes(P, n, 2, args.group, True, variant) if path == "one kernel" else mb["total"]
        print(json.dumps({"sweep": True, "variant": args.variant, "group": args.group, "n_per_rank": n,
                          "msg_bytes": 2 * n, "calls": calls, "path": path, "bytes_per_call": path_bytes,
                          "us_per_call": round(ms * 1e3, 2),
                          "us_per_call_median16": round(ms_median * 1e3, 2),
                          # the call's bytes fit the 126 MB L2: may read above the HBM roofline
                          "l2_resident": mb["total"] < L2_BYTES,
                          "us_per_call_graph": round(ms_graph * 1e3, 2),
                          "algbw_GBs": round(2 * n / (ms * 1e-3) / 1e9, 2),
                          "algbw_graph_GBs": round(2 * n / (ms_graph * 1e-3) / 1e9, 2),
                          "roofline_frac_graph": round(path_bytes / (ms_graph * 1e-3) / (peak * 1e9), 4)}),
              flush=True)
        h.close()


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--sweep", action="store_true",
                    help="print one line per message size (2^12..2^29 elements) instead of the benchmark")
    ap.add_argument("--sweep-max", type=int, default=29, choices=range(12, 30), metavar="K",
                    help="with --sweep: the largest size, 2^K elements per rank (default 29)")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["echo", "reference"], default="echo")
    ap.add_argument("--n", "--elems", dest="n", type=int, default=N_ELEMS,
                    help="elements per rank (default 2^29); under torchrun spell it --elems, which "
                         "torchrun's own options do not abbreviate")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--variant", choices=sorted(VARIANTS), default="default",
                    help="where rounding errors are fed back (default: the method as read)")
    ap.add_argument("--group", type=int, choices=[16, 32, 64, 128], default=32,
                    help="elements per scale (default 32, the method as read)")
    ap.add_argument("--ranks", type=int, default=8, choices=range(2, 17), metavar="P",
                    help="ranks of the all-reduce, 2..16 (default 8, the benchmark's workload)")
    ap.add_argument("--mode", choices=["auto", "simulated", "sharded", "replicas"], default="auto",
                    help="simulated: one handle, ranks in one GPU's HBM; sharded: one handle per rank, "
                         "ranks spread over the processes; replicas: an independent simulated problem "
                         "per GPU (auto: simulated at one process, sharded at more)")
    ap.add_argument("--config", type=int, choices=[1, 2, 4, 5], default=None,
                    help="print one line for this workload instead of the benchmark line")
    ap.add_argument("--fused-limit", type=int, default=None, metavar="N",
                    help="calls with n <= N elements per rank run as one kernel (0: never). Default: the "
                         "library's 2^20 with --config and --sweep; the three kernels on the benchmark line")
    ap.add_argument("--one-gpu", action="store_true",
                    help="sharded mode: every process uses GPU 0 (with --gpus 1)")
    ap.add_argument("--host-ordered", action="store_true",
                    help="sharded mode: synchronise the stream before each stage barrier instead of "
                         "ordering the stages with events")
    args = ap.parse_args(argv)
    global P
    P = args.ranks
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank, world, local = dist_env()
    if args.one_gpu:
        if args.gpus != 1:
            ap.error("--one-gpu runs every process on GPU 0: use it with --gpus 1")
    elif world != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE is {world}")
    mode = args.mode if args.mode != "auto" else ("simulated" if world == 1 else "sharded")
    if mode == "simulated" and world > 1:
        ap.error("simulated mode runs one process; use --mode replicas or sharded")
    if mode == "sharded" and P % world:
        ap.error(f"--ranks {P} does not split evenly over {world} processes")
    if mode != "sharded" and (args.one_gpu or args.host_ordered):
        ap.error("--one-gpu and --host-ordered belong to the sharded mode")

    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0
    if args.sweep:
        if rank == 0:
            run_sweep(args)
        return 0
    if args.config is not None:
        if rank == 0:
            print(json.dumps(run_config(args)), flush=True)
        return 0

    if mode == "sharded":
        res = run_sharded(args, rank, world, local)
    else:
        res = run_echo(args, rank, world, local)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if res is not None:
        if world == 1 and mode == "simulated" and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline_leg(VARIANTS[args.variant])
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
