"""Throughput of the block-sparse causal attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step is one forward pass (one kernel launch) over the workload's whole
batch.  Prints one JSON line on rank 0.

value      useful TFLOP/s = 4 * D * (allowed pairs per head) * B * Hq per step,
           divided by the device time of K steps (CUDA events, barrier and
           synchronize on both sides, max over ranks); inputs resident in HBM.
           Inputs rotate over several sets whose footprint exceeds L2.
roofline   the forward kernel against the measured dense bf16 tensor peak:
           executed-tile FLOP per launch (4 * D * block^2 per live tile) over
           the mean per-launch duration: this rank's K back-to-back launches
           timed with one pair of CUDA events on the launching stream.
e2e        the same metric through the host-buffer C ABI call (pinned host
           Q/K/V and the host mask in, O/LSE out, copies inside the timed
           region), the steps queued back to back (each step's inputs cross
           PCIe while the previous step's outputs come back); the latency of
           one blocking call is reported beside it.
cpu_baseline  the fp64 CPU oracle on a bounded row sample, host cores.

With --pass bwd one step is one backward pass (four launches: work items,
prep, the tensor-core kernel, dQ conversion) for an upstream gradient dO, with the
forward's O and LSE computed once before timing; value counts 10 * D useful
FLOP per allowed pair (S, dP, dV, dK, dQ) and the roofline takes the whole
step's device time (the launch list in profiles/ gives each kernel's share).

With --path stride (patterns with a stride) one step is the stride-aware
forward: three grouping copies, the pattern without its stride in token
order, the remaining stride pairs on tokens grouped by residue, and the merge;
the roofline then counts the executed tiles of both passes over the whole
step's device time.

With --impl reference the oracle is the timed program (rank 0 only).
Multi-GPU (torchrun): every rank runs its own batch of the workload (the
problems are independent; no collective on the data path); value is the sum
over ranks of the work divided by the slowest rank's time ("scaling": "weak").
With --shard heads the ranks split one workload instead: each takes a
contiguous range of its batch x kv-head groups with their query heads, again
with no collective on the data path; value is the workload's work over the
slowest rank's time ("scaling": "strong").
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402
from synth.workloads import HEADLINE, WORKLOADS  # noqa: E402

METRIC = "block-sparse attn fwd useful TFLOP/s (bf16, 1 B200) and % of tensor peak"
METRIC_BWD = "block-sparse attn bwd useful TFLOP/s (bf16, 1 B200) and % of tensor peak"
UNIT = "TFLOP/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
KERNEL_SOURCES = ["block_sparse_attention_build_b200/csrc/fwd_sm100.cuh",
                  "block_sparse_attention_build_b200/csrc/sm100.cuh"]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_sha() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per launch from the committed ncu summary of this workload,
    if it was taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", f"fwd_kernel_{workload}.md")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and line.strip().startswith("- "):
                k, _, v = line.strip()[2:].partition(":")
                vals[k.strip()] = v.strip().strip("`")
    if vals.get("kernel_source_sha") != kernel_sha():
        return None
    try:
        return int(vals["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def workload_counts(w):
    import block_sparse_attention_build_b200 as sa
    p = sa.Pattern(**w.pattern_args())
    pairs = sa.count_pairs(p, w.N)
    mask = sa.build_block_mask(p, w.N, w.block)
    useful = 4.0 * w.D * pairs * w.B * w.Hq
    executed = 4.0 * w.D * w.block * w.block * mask.n_live * w.B * w.Hq
    qo = w.B * w.Hq * w.N * w.D * 2
    kv = w.B * w.Hkv * w.N * w.D * 2
    min_bytes = 2 * qo + 2 * kv + w.B * w.Hq * w.N * 4
    return p, mask, pairs, useful, executed, min_bytes


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""

    FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def _sample_rows(w, n):
    return np.unique(np.linspace(0, w.N - 1, n).round().astype(np.int64))


def _sample_flops(w, rows):
    """Useful FLOP of the sampled rows: 4 * D * (allowed keys of each row) * B * Hq,
    the keys counted by the oracle (the CPU arms never load the CUDA library)."""
    import oracle
    keys = int(oracle.row_counts(oracle.Pattern(**w.pattern_args()), w.N, rows).sum())
    return 4.0 * w.D * keys * w.B * w.Hq


class OracleSample:
    """The fp64 CPU oracle on an evenly spaced row sample of the workload (all
    batches and heads), sized once to about target_s seconds per call."""

    def __init__(self, w, target_s: float):
        import oracle
        self.oracle = oracle
        self.w = w
        self.q, self.k, self.v = synth.qkv(w.B, w.Hq, w.Hkv, w.N, w.D, seed=w.seed)
        self.op = oracle.Pattern(**w.pattern_args())
        n = 8
        while True:
            rows = _sample_rows(w, n)
            dt = self._time(rows)
            if dt >= target_s or n >= w.N:
                break
            n = min(w.N, max(n * 2, int(n * target_s / max(dt, 1e-4) * 1.05)))
        self.rows = rows
        self.flops = _sample_flops(w, rows)
        self.threads = oracle.max_threads()

    def _time(self, rows):
        t0 = time.perf_counter()
        self.oracle.attention(self.q, self.k, self.v, self.op, self.w.scale, rows=rows)
        return time.perf_counter() - t0

    def run(self):
        """One timed call: (useful TFLOP/s, seconds)."""
        dt = self._time(self.rows)
        return self.flops / dt / 1e12, dt

    def describe(self, dt):
        return (f"{len(self.rows)} evenly spaced query rows of {self.w.N} x all {self.w.B * self.w.Hq} "
                f"(batch, head) pairs, fp64, {dt:.2f} s per call")


def run_reference(args, w):
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    if args.which == "bwd":
        # whole heads of the fp64 backward oracle, about 20 s in all
        cpu = oracle_bwd_baseline(w, 20.0)
        line = {
            "impl": "reference", "metric": METRIC_BWD, "value": cpu["value"], "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, args.gpus, {"pass": "bwd"}), "cpu_baseline": cpu,
            "e2e": {"value": cpu["value"], "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line))
        return 0
    per_step = min(2.0, max(0.01, 120.0 / (args.steps + args.warmup)))
    sample = OracleSample(w, per_step)
    for _ in range(args.warmup):
        sample.run()
    secs = [sample.run()[1] for _ in range(args.steps)]
    total = float(np.sum(secs))
    value = sample.flops * args.steps / total / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(w, args.gpus, None if args.path == "plain" else {"path": "stride-aware"},
                                                  shard=args.shard == "heads" and args.gpus > 1),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": sample.threads, "kind": "oracle",
                         "sample": sample.describe(total / args.steps)},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def config_of(w, n_gpus, extra=None, shard=False):
    """The workload as both arms report it (the same dict for the same run)."""
    c = {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "D": w.D,
         "pattern": {"causal": 1, **w.pattern_args()}, "block": w.block, "seed": w.seed,
         "inputs": "iid N(0,1) -> bf16, scale 1/sqrt(D)",
         "l2": f"GPU timing rotates the inputs over up to 8 sets whose footprint exceeds the "
               f"{L2_BYTES / 1e6:.0f} MB L2 (no flush); workload_info.input_sets gives the sets",
         "parallelism": ("single GPU" if n_gpus == 1 else
                         f"kv heads sharded over {n_gpus} GPUs (contiguous ranges of the batch x kv-head "
                         f"groups; no data-path collective)" if shard else
                         f"{n_gpus} independent batches, one per GPU")}
    if extra:
        c.update(extra)
    return c


def shard_heads(n_heads: int, world: int, rank: int):
    """Rank's contiguous range [h0, h1) of the n_heads kv heads (flattened over
    batch and head) when one workload is split across ranks."""
    return n_heads * rank // world, n_heads * (rank + 1) // world


def shard_inputs(q, k, v, B, Hq, Hkv, h0, h1):
    """The rank's part of one workload's inputs: kv heads h0 .. h1 - 1 of the
    flattened batch x head axis and their query heads, as a batch of one."""
    g = Hq // Hkv
    N, D = q.shape[2], q.shape[3]
    qs = q.reshape(B * Hkv, g, N, D)[h0:h1].reshape(1, (h1 - h0) * g, N, D)
    ks = k.reshape(B * Hkv, N, D)[h0:h1].reshape(1, h1 - h0, N, D)
    vs = v.reshape(B * Hkv, N, D)[h0:h1].reshape(1, h1 - h0, N, D)
    return np.ascontiguousarray(qs), np.ascontiguousarray(ks), np.ascontiguousarray(vs)


def rank_seed(w, rank: int) -> int:
    """Every rank runs its own, independent batch of the workload (weak scaling)."""
    return w.seed + rank


def max_over_ranks(value: float, dist, device) -> float:
    """The slowest rank's time: all_reduce(MAX) of a per-rank float (identity at world 1)."""
    import torch
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world: int, flop_per_rank_step: float, steps: int, elapsed_ms: float) -> float:
    """Whole-job throughput: the work of all ranks over the slowest rank's time."""
    return world * flop_per_rank_step * steps / (elapsed_ms * 1e-3) / 1e12


def run_gpu(args, w):
    import torch
    import torch.distributed as dist

    import block_sparse_attention_build_b200 as sa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    p, mask_h, pairs, useful, executed, min_bytes = workload_counts(w)
    mask = mask_h.to_device(dev)
    stride_path = args.path == "stride"
    # the stride-aware path reads pass 2 through grouped views (no copies) when the
    # residue groups (N / stride tokens each) fill whole tiles
    n_group = w.N // max(w.stride, 1)
    grouped_in_place = n_group % 128 == 0 and n_group % w.block == 0
    if stride_path:
        if w.stride <= 0:
            raise SystemExit("--path stride needs a workload with a stride")
        plan_h = sa.stride_plan(p, w.N, w.block)
        plan = tuple(m.to_device(dev) for m in plan_h)
        executed = 4.0 * w.D * w.block * w.block * sum(m.n_live for m in plan_h) * w.B * w.Hq
        if args.shard == "heads" and world > 1:
            raise SystemExit("--shard heads runs the plain path")
        sws = torch.empty(sa.fwd_stride_workspace_bytes(w.B, w.Hq, w.Hkv, w.N, w.D), dtype=torch.uint8,
                          device=dev)

    # inputs: every rank its own batch (seed offset by rank), or with --shard
    # heads its range of the one workload's kv heads; rotate sets past L2
    shard = args.shard == "heads" and world > 1
    if shard:
        if world > w.B * w.Hkv:
            raise SystemExit(f"--shard heads needs at most {w.B * w.Hkv} ranks for {w.name}")
        h0, h1 = shard_heads(w.B * w.Hkv, world, rank)
        q, k, v = shard_inputs(*synth.qkv(w.B, w.Hq, w.Hkv, w.N, w.D, seed=w.seed), w.B, w.Hq, w.Hkv, h0, h1)
        rB, rHkv, rHq = 1, h1 - h0, (h1 - h0) * (w.Hq // w.Hkv)
    else:
        q, k, v = synth.qkv(w.B, w.Hq, w.Hkv, w.N, w.D, seed=rank_seed(w, rank))
        rB, rHkv, rHq = w.B, w.Hkv, w.Hq
    rank_part = rB * rHkv / (w.B * w.Hkv)  # this rank's share of one workload's work
    job_useful = useful if shard else world * useful  # work of the whole job per step
    to_dev = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    set_bytes = min_bytes * rank_part  # this rank's inputs and outputs
    n_sets = args.sets if args.sets > 0 else max(1, min(8, math.ceil(3 * L2_BYTES / set_bytes)))
    Q0, K0, V0 = to_dev(q), to_dev(k), to_dev(v)
    sets = []
    for i in range(n_sets):
        Qi, Ki, Vi = (Q0, K0, V0) if i == 0 else (Q0.clone(), K0.clone(), V0.clone())
        Oi = torch.empty_like(Qi)
        Li = torch.empty((rB, rHq, w.N), dtype=torch.float32, device=dev)
        sets.append((Qi, Ki, Vi, Oi, Li))
    stream = torch.cuda.current_stream(dev)

    def step(i):
        Qi, Ki, Vi, Oi, Li = sets[i % n_sets]
        if stride_path:
            sa.fwd_stride(Qi, Ki, Vi, plan[0], plan[1], p, scale=w.scale, out=Oi, lse=Li, workspace=sws,
                          stream=stream)
        else:
            sa.fwd(Qi, Ki, Vi, mask, p, scale=w.scale, out=Oi, lse=Li, stream=stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    if sa.check_device(stream) != sa.SA_OK:
        raise SystemExit("device status not ok after warm-up")

    # One event pair around the K launches: an event recorded between two launches
    # would end the overlap of one launch's start with the previous one's tail.
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        t_start.record(stream)
        for i in range(args.steps):
            step(i)
        t_end.record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
    elapsed_ms = t_start.elapsed_time(t_end)
    local_elapsed_ms = elapsed_ms
    status = sa.check_device(stream)
    if status != sa.SA_OK:
        raise SystemExit(f"device status {sa.status_string(status)}")
    elapsed_ms = max_over_ranks(elapsed_ms, dist if world > 1 else None, dev)
    mean_launch_ms = local_elapsed_ms / args.steps  # this rank's launches, back to back

    # end to end through the host-buffer entry point (pinned memory)
    e2e = None
    if not args.no_e2e and not stride_path:
        pin = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory()
        Qh, Kh, Vh = pin(q), pin(k), pin(v)
        Oh = torch.empty((rB, rHq, w.N, w.D), dtype=torch.bfloat16).pin_memory()
        Lh = torch.empty((rB, rHq, w.N), dtype=torch.float32).pin_memory()
        ws = torch.empty(sa.fwd_host_workspace_bytes(rB, rHq, rHkv, w.N, w.D), dtype=torch.uint8,
                         device=dev)
        e2e_steps = max(3, min(args.steps, 20))
        for _ in range(2):
            sa.fwd_host(Qh, Kh, Vh, mask_h, p, Oh, Lh, ws, scale=w.scale, stream=stream)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        # one blocking call per step: its latency
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(3):
            sa.fwd_host(Qh, Kh, Vh, mask_h, p, Oh, Lh, ws, scale=w.scale, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        sync_ms = e0.elapsed_time(e1) / 3
        # the steps queued back to back: each step's inputs cross PCIe while the
        # previous step's outputs come back; one wait at the end
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(e2e_steps):
            sa.fwd_host(Qh, Kh, Vh, mask_h, p, Oh, Lh, ws, scale=w.scale, stream=stream, wait=False)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        if sa.check_device(stream) != sa.SA_OK:
            raise SystemExit("device status not ok after the end-to-end leg")
        e2e_ms = e0.elapsed_time(e1)
        e2e_ms = max_over_ranks(e2e_ms, dist if world > 1 else None, dev)
        h2d = sum(t.numel() * t.element_size() for t in (Qh, Kh, Vh))
        h2d += sum(a.nbytes for a in (mask_h.counts, mask_h.index, mask_h.full))  # the host block mask
        d2h = Oh.numel() * Oh.element_size() + Lh.numel() * Lh.element_size()
        e2e = {"value": job_tflops(1, job_useful, e2e_steps, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
               "ms_per_step": e2e_ms / e2e_steps, "api": "sparse_attn_fwd_host_async, steps queued back to back",
               "blocking_call_ms": sync_ms}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks, peak_kind = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    value = job_tflops(1, job_useful, args.steps, elapsed_ms)
    achieved = executed * rank_part / (mean_launch_ms * 1e-3) / 1e12  # rank 0's kernel
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        sample = OracleSample(w, args.cpu_seconds)
        rate, dt = sample.run()
        cpu = {"value": rate, "unit": UNIT, "cores": sample.threads, "kind": "oracle",
               "sample": sample.describe(dt)}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
        "scaling": "strong" if shard else "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_of(w, world, {"path": "stride-aware"} if stride_path else None, shard=shard),
        "workload_info": {
            "input_sets": f"{n_sets} of {set_bytes / 1e6:.1f} MB per rank",
            "live_tiles": int(mask_h.n_live), "full_tiles": int(mask_h.n_full),
            "allowed_pairs_per_head": int(pairs),
            **({"executed_tiles_per_head": int(sum(m.n_live for m in plan_h))} if stride_path else {})},
        "useful_frac_of_peak": value / world / peak,
        "executed_tflops": job_tflops(1, executed if shard else world * executed, args.steps, elapsed_ms),
        "executed_frac_of_peak": executed * rank_part / (elapsed_ms / args.steps * 1e-3) / 1e12 / peak,
        "peak_kind": f"bf16 dense, {peak_kind} ({peak} TFLOP/s burst)",
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": None if stride_path else profiled_traffic(w.name),
                     "kernel": (("stride-aware step: 2 x fwd_kernel + merge"
                                 + ("" if grouped_in_place else " + 3 grouping copies")) if stride_path
                                else "fwd_kernel<D,BN>"),
                     "mean_launch_us": mean_launch_ms * 1e3,
                     "algorithmic_flop_per_launch": executed,
                     "hbm_gbs_min_bytes": min_bytes / (mean_launch_ms * 1e-3) / 1e9},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": args.steps * ((3 if grouped_in_place else 6) if stride_path else 1),
        "clocks": clocks.summary(),
    }
    print(json.dumps(line))
    return 0


def run_gpu_bwd(args, w):
    """The backward pass of the workload: one step = sparse_attn_bwd over the batch."""
    import torch
    import torch.distributed as dist

    import block_sparse_attention_build_b200 as sa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    p, mask_h, pairs, _, _, _ = workload_counts(w)
    useful = 10.0 * w.D * pairs * w.B * w.Hq
    mask = mask_h.to_device(dev)
    # The backward works on 128 x 128 tiles whatever tile the forward used: it
    # takes the transposed block-128 mask of the same pattern (partial tiles are
    # masked element by element from the rule, so the gradients are the same).
    mask128 = mask_h if w.block == 128 else sa.build_block_mask(p, w.N, 128)
    executed = 10.0 * w.D * 128 * 128 * mask128.n_live * w.B * w.Hq
    mask_t = sa.transpose_block_mask(mask128).to_device(dev)

    seed = rank_seed(w, rank)
    q, k, v = synth.qkv(w.B, w.Hq, w.Hkv, w.N, w.D, seed=seed)
    do = synth.qkv(w.B, w.Hq, w.Hkv, w.N, w.D, seed=seed + 7919)[0]
    to_dev = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    Q0, K0, V0, dO0 = to_dev(q), to_dev(k), to_dev(v), to_dev(do)
    O0, L0 = sa.fwd(Q0, K0, V0, mask, p, scale=w.scale)
    ws_bytes = sa.bwd_workspace_bytes(w.B, w.Hq, w.Hkv, w.N, w.D)
    qo = w.B * w.Hq * w.N * w.D * 2
    kv = w.B * w.Hkv * w.N * w.D * 2
    set_bytes = 4 * qo + 4 * kv + w.B * w.Hq * w.N * 4 + ws_bytes  # Q O dO dQ, K V dK dV, LSE, workspace
    n_sets = args.sets if args.sets > 0 else max(2, min(8, math.ceil(3 * L2_BYTES / set_bytes)))
    sets = []
    for i in range(n_sets):
        ins = (Q0, K0, V0, O0, L0, dO0) if i == 0 else tuple(t.clone() for t in (Q0, K0, V0, O0, L0, dO0))
        outs = (torch.empty_like(Q0), torch.empty_like(K0), torch.empty_like(V0),
                torch.empty(ws_bytes, dtype=torch.uint8, device=dev))
        sets.append((ins, outs))
    stream = torch.cuda.current_stream(dev)

    def step(i):
        (Qi, Ki, Vi, Oi, Li, dOi), (dQi, dKi, dVi, Wi) = sets[i % n_sets]
        sa.bwd(Qi, Ki, Vi, Oi, Li, dOi, mask_t, p, scale=w.scale, dq=dQi, dk=dKi, dv=dVi, workspace=Wi,
               stream=stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    if sa.check_device(stream) != sa.SA_OK:
        raise SystemExit("device status not ok after warm-up")
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        t_start.record(stream)
        for i in range(args.steps):
            step(i)
        t_end.record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
    local_ms = t_start.elapsed_time(t_end)
    status = sa.check_device(stream)
    if status != sa.SA_OK:
        raise SystemExit(f"device status {sa.status_string(status)}")
    elapsed_ms = max_over_ranks(local_ms, dist if world > 1 else None, dev)
    step_ms = local_ms / args.steps

    # end to end: pinned host inputs in, gradients out, every step
    e2e = None
    if not args.no_e2e:
        pin = lambda t: t.cpu().pin_memory()
        hins = [pin(t) for t in (Q0, K0, V0, O0, L0, dO0)]
        houts = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (Q0, K0, V0)]
        dins = [torch.empty_like(t) for t in (Q0, K0, V0, O0, L0, dO0)]
        douts = [torch.empty_like(t) for t in (Q0, K0, V0)]
        W = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)

        def e2e_step():
            for d, h in zip(dins, hins):
                d.copy_(h, non_blocking=True)
            sa.bwd(*dins, mask_t, p, scale=w.scale, dq=douts[0], dk=douts[1], dv=douts[2], workspace=W,
                   stream=stream)
            for h, d in zip(houts, douts):
                h.copy_(d, non_blocking=True)

        e2e_steps = max(3, min(args.steps, 20))
        for _ in range(2):
            e2e_step()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist if world > 1 else None, dev)
        e2e = {"value": job_tflops(world, useful, e2e_steps, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in hins),
               "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in houts), "steps": e2e_steps,
               "ms_per_step": e2e_ms / e2e_steps}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    peaks, peak_kind = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    value = job_tflops(world, useful, args.steps, elapsed_ms)
    achieved = executed / (step_ms * 1e-3) / 1e12
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = oracle_bwd_baseline(w, args.cpu_seconds)
    line = {
        "metric": METRIC_BWD, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_of(w, world, {"pass": "bwd"}),
        "workload_info": {"input_sets": f"{n_sets} of {set_bytes / 1e6:.1f} MB",
                          "live_tiles": int(mask128.n_live), "backward_tile": 128,
                          "allowed_pairs_per_head": int(pairs)},
        "useful_frac_of_peak": value / world / peak,
        "executed_tflops": job_tflops(world, executed, args.steps, elapsed_ms),
        "peak_kind": f"bf16 dense, {peak_kind} ({peak} TFLOP/s burst)",
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": None,
                     "kernel": "backward step: bwd_items_kernel + bwd_prep_kernel + bwd_kernel<D> + bwd_dq_kernel",
                     "mean_step_us": step_ms * 1e3, "algorithmic_flop_per_step": executed},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": 4 * args.steps,
        "clocks": clocks.summary(),
    }
    print(json.dumps(line))
    return 0


def oracle_bwd_baseline(w, target_s: float):
    """The fp64 backward oracle on whole heads of the workload (host cores),
    as many heads as fit in about target_s seconds (at least one)."""
    import oracle
    p = oracle.Pattern(**w.pattern_args())
    q, k, v = synth.qkv(1, 1, 1, w.N, w.D, seed=w.seed)
    do = synth.qkv(1, 1, 1, w.N, w.D, seed=w.seed + 7919)[0]
    pairs = oracle.count_pairs(p, w.N)
    heads, t0 = 0, time.perf_counter()
    while True:
        oracle.attention_bwd(q, k, v, do, p, w.scale)
        heads += 1
        dt = time.perf_counter() - t0
        if dt >= target_s or dt / heads * (heads + 1) > 2 * target_s:
            break
    rate = 10.0 * w.D * pairs * heads / dt / 1e12
    return {"value": rate, "unit": UNIT, "cores": oracle.max_threads(), "kind": "oracle",
            "sample": f"{heads} whole head(s) of N={w.N} (dQ, dK, dV in fp64), {dt:.1f} s"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer leg (profiling runs)")
    ap.add_argument("--sets", type=int, default=0, help="rotating input sets (0: enough to exceed L2)")
    ap.add_argument("--pass", dest="which", default="fwd", choices=["fwd", "bwd"])
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads"],
                    help="with several GPUs: every rank its own batch (weak scaling), or one workload's "
                         "kv heads split across the ranks (strong scaling)")
    ap.add_argument("--path", default="plain", choices=["plain", "stride"],
                    help="forward path: one block-sparse kernel, or the stride-aware two-pass path")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    if args.which == "bwd":
        return run_gpu_bwd(args, w)
    return run_gpu(args, w)


if __name__ == "__main__":
    sys.exit(main())
