"""Benchmark of the Monarch attention forward (one call = one step).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload: the full-clip video latent, B=1, 12 heads, d=128, T=21 frames of
30x52 tokens (N=32760), frame-aligned factorisation (m=1560, b=21), bf16,
seeded synthetic inputs (see structured_attention_video_monarch_b200/workloads.py).
Metric: effective TFLOP/s counting 4*N*(m+b)*d FLOPs per (batch, head), plus
ms per call and the fraction of the measured B200 bf16 dense peak.

Our arm times K calls with CUDA events on the launching stream, bracketed by a
barrier and a device synchronisation, and reports the max over ranks.  Each
rank runs its own full workload (the operator shards over independent
(batch, head) problems with no collective, so N GPUs run N replicas: weak
scaling).  Between timed calls the inputs rotate over three buffer sets
(1.2 GB in all), so every call reads inputs that are not resident in the
126 MB L2.  The reference arm (--impl reference) times the fp64 CPU oracle on
a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import tempfile
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "Monarch attn fwd ms & effective TFLOP/s at N=32760; % of B200 bf16 peak"
WORKLOAD = "fullclip_bf16"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def workload_config(wl, extra=None):
    cfg = {
        "workload": (f"{wl.name}: B={wl.B} heads={wl.heads} d={wl.d} T={wl.T} H={wl.H} W={wl.W} "
                     f"(N={wl.N}), "
                     f"{('frame', 'tiled ' + str(wl.tile_h) + 'x' + str(wl.tile_w), '(f*h, w)')[wl.fact]}"
                     f" split m={wl.m} b={wl.b}"
                     + (f"; chunk of {wl.T} new frames after {wl.T_ctx} context frames" if wl.T_ctx else "")),
        "global_batch": wl.B,
        "seq_len": wl.N,
        "heads": wl.heads,
        "head_dim": wl.d,
        "flops_per_call": wl.flops,
    }
    if extra:
        cfg.update(extra)
    return cfg


# ------------------------------------------------------------------ distributed helpers

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def aggregate(world: int, flops_per_call: float, steps: int, max_seconds: float):
    """Whole-job throughput: all ranks' FLOPs over the slowest rank's time."""
    total = world * flops_per_call * steps
    return total / max_seconds / 1e12, max_seconds * 1e3 / steps


# ------------------------------------------------------------------ clock sampling

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, log_dir: str | None = None):
        self.index = index
        self.proc = None
        self.keep = bool(log_dir)
        if log_dir:  # keep the raw samples
            self.path = os.path.join(log_dir, f"clocks_rank{index}.csv")
        else:
            fd, self.path = tempfile.mkstemp(prefix=f"clocks_rank{index}_", suffix=".csv")
            os.close(fd)

    def start(self):
        os.makedirs(os.path.dirname(self.path) or ".", exist_ok=True)
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            if not self.keep and os.path.exists(self.path):
                os.unlink(self.path)
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as fh:
            lines = fh.readlines()
        if not self.keep:
            os.unlink(self.path)
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[4:]))
            except ValueError:
                continue
        if not rows:
            return None
        load = [r for r in rows if r[2] > 300.0] or rows  # samples under load (power draw)
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in load:
            for name, flag in zip(names, r[3][1:]):
                if flag.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r[0] for r in load), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows), "samples_under_load": len(load)}


# ------------------------------------------------------------------ CPU baseline (oracle)

def oracle_sample(wl, seconds: float, seed: int = 1234):
    """Time the fp64 oracle on a bounded sample: G whole stage-2 groups (each =
    T output rows with their exact stage-1 rows), sized to about `seconds`."""
    import numpy as np
    import oracle
    from structured_attention_video_monarch_b200 import workloads
    q, k, v = workloads.generate(wl, heads=1)  # one head's problem, same shape per head
    HW = wl.H * wl.W
    flops_per_group = 4.0 * wl.T * (wl.m + wl.b) * wl.d
    rng = np.random.default_rng(seed)
    g = 8
    t0 = time.perf_counter()
    oracle.monarch_fwd_groups(q, k, v, wl.T, wl.H, wl.W,
                              [(0, int(p)) for p in rng.integers(0, HW, g)], wl.fact, wl.tile_h, wl.tile_w)
    dt = time.perf_counter() - t0
    g = max(8, min(HW, int(g * seconds / max(dt, 1e-6))))
    groups = [(0, int(p)) for p in rng.integers(0, HW, g)]
    return q, k, v, groups, flops_per_group


def oracle_chunk_sample(wl, seconds: float):
    """Time the fp64 oracle's chunk form on whole heads of a chunk workload:
    as many heads (one call each) as fit in about `seconds`.  Returns
    (TFLOP/s, seconds, heads)."""
    import oracle
    from structured_attention_video_monarch_b200 import workloads
    q, k, v = workloads.generate(wl, heads=1)
    kc, yc = workloads.generate_context(wl, heads=1)
    args = [x.double().numpy() for x in (q, k, v, kc, yc)]

    def one():
        oracle.monarch_fwd_chunk(*args, wl.T_ctx, wl.T, wl.H, wl.W, wl.fact, wl.tile_h, wl.tile_w)

    t0 = time.perf_counter()
    one()
    dt1 = time.perf_counter() - t0
    reps = max(1, min(wl.heads * wl.B, int(seconds / max(dt1, 1e-6))))
    t0 = time.perf_counter()
    for _ in range(reps):
        one()
    dt = time.perf_counter() - t0
    per_head = wl.flops / (wl.B * wl.heads)
    return reps * per_head / dt / 1e12, dt, reps


def oracle_head_sample(wl, seconds: float):
    """Time the fp64 oracle's full forward on whole heads (for the (f*h, w)
    split, whose column groups span every frame, so no exact sampled-group
    form exists): as many heads (one call each) as fit in about `seconds`.
    Returns (TFLOP/s, seconds, heads)."""
    import oracle
    from structured_attention_video_monarch_b200 import workloads
    q, k, v = (x.double().numpy() for x in workloads.generate(wl, heads=1))

    def one():
        oracle.monarch_fwd(q, k, v, wl.T, wl.H, wl.W, wl.fact, wl.tile_h, wl.tile_w)

    t0 = time.perf_counter()
    one()
    dt1 = time.perf_counter() - t0
    reps = max(1, min(wl.heads * wl.B, int(seconds / max(dt1, 1e-6))))
    t0 = time.perf_counter()
    for _ in range(reps):
        one()
    dt = time.perf_counter() - t0
    per_head = wl.flops / (wl.B * wl.heads)
    return reps * per_head / dt / 1e12, dt, reps


def oracle_bwd_sample(wl, seconds: float):
    """Time the fp64 gradient oracle on whole heads of a gradient workload:
    as many heads (one call each) as fit in about `seconds`.  Returns
    (TFLOP/s, seconds, heads)."""
    import oracle
    from structured_attention_video_monarch_b200 import workloads
    q, k, v = (x.double().numpy() for x in workloads.generate(wl, heads=1))
    do = workloads.generate_upstream(wl, heads=1).double().numpy()

    def one():
        oracle.monarch_bwd(q, k, v, do, wl.T, wl.H, wl.W, wl.fact, wl.tile_h, wl.tile_w)

    t0 = time.perf_counter()
    one()
    dt1 = time.perf_counter() - t0
    reps = max(1, min(wl.heads * wl.B, int(seconds / max(dt1, 1e-6))))
    t0 = time.perf_counter()
    for _ in range(reps):
        one()
    dt = time.perf_counter() - t0
    per_head = wl.flops / (wl.B * wl.heads)
    return reps * per_head / dt / 1e12, dt, reps


def time_oracle(wl, q, k, v, groups, flops_per_group):
    import oracle
    t0 = time.perf_counter()
    oracle.monarch_fwd_groups(q, k, v, wl.T, wl.H, wl.W, groups, wl.fact, wl.tile_h, wl.tile_w)
    dt = time.perf_counter() - t0
    return len(groups) * flops_per_group / dt / 1e12, dt


def run_reference(args):
    import oracle
    from structured_attention_video_monarch_b200 import workloads
    rank, _, world = dist_env()
    wl = workloads.BY_NAME[args.workload]
    if rank != 0:
        return 0
    oracle.build()
    budget = max(0.5, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    if wl.T_ctx or wl.grad or wl.fact == workloads.FACT_ROW:
        return run_reference_heads(args, wl, budget)
    q, k, v, groups, fpg = oracle_sample(wl, budget)
    for _ in range(args.warmup):
        time_oracle(wl, q, k, v, groups, fpg)
    total = 0.0
    for _ in range(args.steps):
        _, dt = time_oracle(wl, q, k, v, groups, fpg)
        total += dt
    value = args.steps * len(groups) * fpg / total / 1e12
    sample = (f"{len(groups)} stage-2 groups x {wl.T} rows of one head per step "
              f"(exact stage-1 + stage-2 rows, {len(groups) * fpg / 1e9:.2f} GFLOP)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, {"parallelism": "host cores (OpenMP)"}),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_reference_heads(args, wl, budget):
    """Reference arm for workloads the oracle times by whole heads: an
    autoregressive chunk, or the (f*h, w) split."""
    import oracle
    sampler = oracle_chunk_sample if wl.T_ctx else (oracle_bwd_sample if wl.grad else oracle_head_sample)
    for _ in range(args.warmup):
        sampler(wl, budget)
    total, flops, heads = 0.0, 0.0, 0
    for _ in range(args.steps):
        val, dt, reps = sampler(wl, budget)
        total += dt
        flops += val * dt * 1e12
        heads = reps
    value = flops / total / 1e12
    if wl.T_ctx:
        sample = (f"{heads} head(s) of the chunk per step (exact stage 1 of the new frames and stage 2 "
                  f"over {wl.T_ctx}+{wl.T} frames)")
    elif wl.grad:
        sample = f"{heads} head(s) of the fp64 gradients (dQ, dK, dV) per step"
    else:
        sample = f"{heads} head(s) of the full forward per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, {"parallelism": "host cores (OpenMP)"}),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm

# The sources each profiled kernel and its launch are built from: whole files,
# or "file#region" for the text between "// <region>" and "// </region>".
KERNEL_SOURCES = {
    "monarch_tc_kernel": ("attn_tc.cuh", "sm100.cuh", "monarch_attn.cu#tc-launch"),
    "monarch_chunk_stage2": ("attn_chunk_mma.cuh", "attn_chunk.cuh", "monarch_attn.cu#chunk-launch"),
    # the tensor-core backward's per-stage phases (row sums, dQ kernel, dK/dV kernel)
    "monarch_bwd_tc_stage1": ("attn_bwd_tc.cuh", "sm100.cuh", "monarch_attn.cu#bwd-launch"),
    "monarch_bwd_tc_stage2": ("attn_bwd_tc.cuh", "sm100.cuh", "monarch_attn.cu#bwd-launch"),
}


def kernel_sources_sha256(kernel: str = "monarch_tc_kernel") -> str:
    """Hash of the CUDA sources a kernel and its launch are built from."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "structured_attention_video_monarch_b200", "csrc")
    for spec in KERNEL_SOURCES[kernel]:
        name, _, region = spec.partition("#")
        with open(os.path.join(csrc, name), "rb") as f:
            text = f.read()
        if region:
            begin, end = f"// <{region}>".encode(), f"// </{region}>".encode()
            i, j = text.find(begin), text.find(end)
            if i < 0 or j < i:
                raise ValueError(f"region {region} not found in {name}")
            text = text[i:j]
        h.update(spec.encode())
        h.update(text)
    return h.hexdigest()


def profile_name(workload: str, kernel: str, part: str | None = None) -> str:
    """Committed ncu summary of a kernel on a workload (one launch or pass of it)."""
    return f"{kernel}_{workload}{'_' + part if part else ''}.md"


def traffic_source(workload: str, kernel: str = "monarch_tc_kernel", part: str | None = None) -> str:
    """Where roofline.traffic comes from, or why it is null."""
    rel = os.path.join("profiles", profile_name(workload, kernel, part))
    if not os.path.exists(os.path.join(ROOT, rel)):
        return "none: no ncu summary for this kernel and workload"
    if captured_traffic(workload, kernel, part) is None:
        return (f"none: {rel} was taken on earlier sources (its kernel_sources_sha256 does not match "
                "the current ones), so its DRAM counters are not reported")
    return f"{rel} (dram__bytes_read.sum + dram__bytes_write.sum of one launch)"


def captured_traffic(workload: str, kernel: str = "monarch_tc_kernel", part: str | None = None):
    """DRAM bytes per launch of `kernel` from the committed ncu summary of this
    workload, or None when there is none or the kernel's sources changed since
    it was taken."""
    path = os.path.join(ROOT, "profiles", profile_name(workload, kernel, part))
    if not os.path.exists(path):
        return None
    fields = {}
    with open(path) as f:
        for line in f:
            key, sep, val = line.strip().partition(":")
            if sep and key in ("kernel_sources_sha256", "traffic_bytes_per_launch"):
                fields[key] = val.strip()
    if fields.get("kernel_sources_sha256") != kernel_sources_sha256(kernel):
        return None
    try:
        return float(fields["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def run_ours(args):
    import torch
    import torch.distributed as dist
    from structured_attention_video_monarch_b200 import binding, workloads

    rank, local_rank, world = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (B200)")
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)
    binding.load_library()
    wl = workloads.BY_NAME[args.workload]
    peaks, peak_src = load_peaks()

    grad = wl.grad        # gradients: dQ, dK, dV of an upstream dO (fp32 path)
    chunk = wl.T_ctx > 0  # autoregressive chunk: new frames plus a resident context
    row = wl.fact == workloads.FACT_ROW  # (f*h, w) split: a rows pass, then a columns pass
    q0, k0, v0 = workloads.generate(wl)
    nsets = 3
    sets = []
    for sidx in range(nsets):
        if sidx == 0:
            q, k, v = q0, k0, v0
        else:  # same distribution, different seed: distinct buffers so L2 holds none of them
            q, k, v = workloads.generate(wl, seed=wl.index + 100 * sidx)
        bufs = tuple(x.to(device) for x in (q, k, v)) + (torch.empty_like(q0, device=device),)
        if chunk:
            ctx = workloads.generate_context(wl, seed=1000 + wl.index + 100 * sidx)
            bufs += tuple(x.to(device) for x in ctx) + (torch.empty_like(q0, device=device),)
        if grad:
            do = workloads.generate_upstream(wl, seed=2000 + wl.index + 100 * sidx).to(device)
            bufs += (do, torch.empty_like(q0, device=device), torch.empty_like(q0, device=device),
                     binding.monarch_attn_bwd_workspace(bufs[0], wl.T, wl.H, wl.W))
        sets.append(bufs)
    stream = torch.cuda.current_stream(device)

    grad16 = grad and wl.dtype != "f32"  # tensor-core gradients: four timed phases

    def call(i, events=None):
        if grad:
            q, k, v, dq, do, dk, dv, ws = sets[i % nsets]
            if grad16:
                if events is None:
                    binding.monarch_attn_bwd(q, k, v, do, wl.T, wl.H, wl.W, wl.fact, wl.tile_h, wl.tile_w,
                                             out=(dq, dk, dv), workspace=ws)
                    return 6  # 2 recomputations, 2 x (row sums, dQ and dK/dV in one launch)
                binding.monarch_attn_bwd_profiled(q, k, v, do, dq, dk, dv, ws, wl.T, wl.H, wl.W, events,
                                                  wl.fact, wl.tile_h, wl.tile_w)
                return 6
            if events is not None:
                events[0].record(stream)
            binding.monarch_attn_bwd(q, k, v, do, wl.T, wl.H, wl.W, wl.fact, wl.tile_h, wl.tile_w,
                                     out=(dq, dk, dv), workspace=ws)
            if events is not None:
                events[1].record(stream)
            return 3  # stage-1 recompute, stage-2 backward, stage-1 backward
        if chunk:
            q, k, v, o, kc, yc, y1 = sets[i % nsets]
            if events is None:
                binding.monarch_attn_fwd_chunk(q, k, v, kc, yc, wl.T_ctx, wl.T, wl.H, wl.W, wl.fact,
                                               wl.tile_h, wl.tile_w, out=o, y1_new=y1)
                return 2
            return binding.monarch_attn_fwd_chunk_profiled(q, k, v, kc, yc, o, y1, wl.T_ctx, wl.T, wl.H,
                                                           wl.W, events, wl.fact, wl.tile_h, wl.tile_w)
        q, k, v, o = sets[i % nsets][:4]
        if events is None:
            binding.monarch_attn_fwd(q, k, v, wl.T, wl.H, wl.W, wl.fact, wl.tile_h, wl.tile_w, out=o)
            return 1
        return binding.monarch_attn_fwd_profiled(q, k, v, o, wl.T, wl.H, wl.W, events, wl.fact,
                                                 wl.tile_h, wl.tile_w)

    for i in range(max(3, args.warmup)):
        call(i)
    torch.cuda.synchronize(device)

    # clocks under load: sample during a short soak of the same calls, then the timed region
    sampler = ClockSampler(device.index, args.clock_log)
    sampler.start()
    t_soak = time.perf_counter()
    i = 0
    while time.perf_counter() - t_soak < args.soak_seconds:
        call(i)
        i += 1
        if i % 50 == 0:
            torch.cuda.synchronize(device)
    torch.cuda.synchronize(device)

    # timed region: K calls, events around each kernel launch
    nev = 5 if grad16 else 3
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(args.steps)]
    for e in (x for row in ev for x in row):
        e.record(stream)  # torch creates the CUDA event on first record; the library needs the handle
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(device)
    torch.cuda.synchronize(device)
    launches = 0
    per_call = []
    start.record(stream)
    for s in range(args.steps):
        n = call(s, ev[s])
        per_call.append(n)
        launches += n
    stop.record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    clocks = sampler.stop()
    elapsed_s = start.elapsed_time(stop) / 1e3
    max_s = max_over_ranks(elapsed_s, device)
    value, ms = aggregate(world, wl.flops, args.steps, max_s)

    # the same calls on one buffer set, back to back, so whatever of the inputs
    # fits in L2 stays there (the timed region above rotates three sets larger
    # than L2); reported beside the main number, not instead of it
    warm = None
    if args.warm_steps > 0:
        for _ in range(3):
            call(0)
        w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(device)
        torch.cuda.synchronize(device)
        w0.record(stream)
        for _ in range(args.warm_steps):
            call(0)
        w1.record(stream)
        torch.cuda.synchronize(device)
        warm_s = max_over_ranks(w0.elapsed_time(w1) / 1e3, device)
        warm_val, warm_ms = aggregate(world, wl.flops, args.warm_steps, warm_s)
        warm = {"value": warm_val, "unit": "TFLOP/s", "ms_per_step": warm_ms, "steps": args.warm_steps,
                "inputs": "one buffer set reused (L2 warm where it fits)"}

    # roofline of the dominant kernel, timed per launch with events on this
    # stream.  The forward is one persistent kernel running both stages; its
    # algorithmic work is the metric's 4*N*(m+b)*d FLOPs per (batch, head).  A
    # chunk is two launches: stage 1 of the new frames (tensor cores) and the
    # stage 2 over context plus new frames (CUDA cores); each is rated
    # against its own work and the slower one is reported as dominant.
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    # the bound follows the arithmetic intensity against the ridge point of
    # the measured peaks (about 247 FLOP/B): the frame split is far above it
    # (tensor cores), small tiles and the chunk's stage 2 fall below it (HBM)
    ridge = peak * 1e12 / (hbm_peak * 1e9)

    # FP32 FMA peak from unit counts and the boost clock: 148 SMs x 128 lanes x 2 FLOP
    # x 1.965 GHz (nothing measured applies to CUDA-core FFMA work)
    alu_peak = 148 * 128 * 2 * float(peaks.get("sm_max_mhz", 1965.0)) * 1e6 / 1e12

    def rate(kernel, label, launch_idx, flops, io_bytes, alu=False, part=None):
        per = sorted(ev[i][launch_idx].elapsed_time(ev[i][launch_idx + 1]) for i in range(args.steps))
        k_avg = statistics.mean(per) / 1e3

        def pct(f):  # nearest-rank percentile of the per-launch times, ms
            return per[min(len(per) - 1, max(0, int(round(f * (len(per) - 1)))))]

        k_tflops = flops / k_avg / 1e12
        k_gbs = io_bytes / k_avg / 1e9
        tensor_bound = flops / io_bytes >= ridge
        traffic = captured_traffic(wl.name, kernel, part)
        t_src = traffic_source(wl.name, kernel, part)
        if args.traffic is not None and launch_idx == 0 and not chunk:
            traffic, t_src = args.traffic, "--traffic argument"
        if alu:
            bound, achieved, pk, unit = "alu", k_tflops, alu_peak, "TFLOP/s"
            src = "derived FP32 FMA peak (148 SMs x 128 lanes x 2 x max SM clock)"
        elif tensor_bound:
            bound, achieved, pk, unit = "tensor", k_tflops, peak, "TFLOP/s"
            src = f"{peak_src} bf16_tflops (burst)"
        else:
            bound, achieved, pk, unit = "hbm", k_gbs, hbm_peak, "GB/s"
            src = f"{peak_src} hbm_gbs (copy)"
        return {
            "bound": bound,
            "achieved": achieved,
            "peak": pk,
            "unit": unit,
            "frac": achieved / pk,
            "traffic": traffic,
            "traffic_source": t_src,
            "kernel": label,
            "peak_source": src,
            "arithmetic_intensity_flop_per_byte": flops / io_bytes,
            "ridge_flop_per_byte": ridge,
            "tflops": k_tflops,
            "tensor_frac": k_tflops / peak,
            "frac_of_sustained": k_tflops / peak_sus,
            "algorithmic_flops_per_launch": flops,
            "launch_ms": k_avg * 1e3,
            "launch_ms_p10_p50_p90": [pct(0.1), pct(0.5), pct(0.9)],
            "algorithmic_bytes_per_launch": io_bytes,
            "hbm_gbs_at_algorithmic_bytes": k_gbs,
            "hbm_frac": k_gbs / hbm_peak,
            "launches_per_call": per_call[0] if per_call else None,
        }

    if grad16:
        # phases: 0 Y1 recompute, 1 O recompute, 2 stage-2 backward, 3 stage-1 backward (writes the outputs).
        # The stage-1 backward (row sums, the dQ kernel and the dK/dV kernel over
        # frame blocks) carries 10*d FLOPs per (query, key) pair of the blocks.
        es, bhd = 2, wl.B * wl.heads * wl.d
        # bytes: read Q, K, V, dY1, Y1 (16-bit) and stage 2's dQ, dK parts (fp32); write dQ, dK, dV (16-bit)
        b1 = rate("monarch_bwd_tc_stage1", f"bwd_rowdot + monarch_bwd_pair<{wl.d}> (dQ and dK/dV CTAs; stage-1 blocks of "
                  f"m={wl.m})", 3, 10.0 * wl.N * wl.m * bhd, (5 * es + 2 * 4 + 3 * es) * wl.N * bhd)
        b2 = rate("monarch_bwd_tc_stage2", f"bwd_rowdot + monarch_bwd_pair<{wl.d}> (dQ and dK/dV CTAs; stage-2 groups of "
                  f"b={wl.b})", 2, 10.0 * wl.N * wl.b * bhd, (5 * es + 2 * 4 + es) * wl.N * bhd)
        phase_ms = {}
        for name, idx in (("recompute_y1", 0), ("recompute_o", 1), ("stage2_bwd", 2), ("stage1_bwd", 3)):
            phase_ms[name] = statistics.mean(ev[i][idx].elapsed_time(ev[i][idx + 1]) for i in range(args.steps))
        roofline = dict(b1, other_kernel=b2, phases_ms=phase_ms)
    elif grad:
        roofline = rate("monarch_bwd_f32", f"monarch_attn_bwd fp32 (3 CUDA-core kernels, d={wl.d}; whole call)",
                        0, wl.flops, wl.io_bytes, alu=True)
    elif row:
        es, bhd = 2, wl.B * wl.heads * wl.d
        r1 = rate("monarch_tc_kernel", f"monarch_tc_kernel<{wl.d}> (rows pass: blocks of W={wl.W} tokens)", 0,
                  4.0 * wl.N * wl.W * bhd, 4 * wl.N * bhd * es, part="rows")
        r2 = rate("monarch_tc_kernel",
                  f"monarch_tc_kernel<{wl.d}> (columns pass: groups of T*H={wl.T * wl.H} tokens)", 1,
                  4.0 * wl.N * wl.T * wl.H * bhd, 4 * wl.N * bhd * es, part="columns")
        roofline, other = (r1, r2) if r1["launch_ms"] >= r2["launch_ms"] else (r2, r1)
        roofline = dict(roofline, other_kernel=other)
    elif chunk:
        es, bhd = 2, wl.B * wl.heads * wl.d
        s1 = rate("monarch_tc_kernel", f"monarch_tc_kernel<{wl.d}> (stage 1 of the {wl.T} new frames)", 0,
                  4.0 * wl.N * wl.m * bhd, 4 * wl.N * bhd * es)
        s2 = rate("monarch_chunk_stage2", f"monarch_chunk_stage2<{wl.d}> (stage 2 over {wl.T_ctx}+{wl.T} frames)",
                  1, 4.0 * wl.N * wl.b * bhd, (4 * wl.N + 2 * wl.N_ctx) * bhd * es)
        roofline, other = (s1, s2) if s1["launch_ms"] >= s2["launch_ms"] else (s2, s1)
        roofline = dict(roofline, other_kernel=other)
    elif wl.dtype == "f32":
        # the exact path: stage 1 and stage 2 are separate CUDA-core launches
        es, bhd = 4, wl.B * wl.heads * wl.d
        f1 = rate("monarch_f32_stage1", f"monarch_f32_stage1<{wl.d}> (stage 1, CUDA cores)", 0,
                  4.0 * wl.N * wl.m * bhd, 4 * wl.N * bhd * es, alu=True)
        f2 = rate("monarch_f32_stage2", f"monarch_f32_stage2<{wl.d}> (stage 2, CUDA cores)", 1,
                  4.0 * wl.N * wl.b * bhd, 4 * wl.N * bhd * es, alu=True)
        roofline, other = (f1, f2) if f1["launch_ms"] >= f2["launch_ms"] else (f2, f1)
        roofline = dict(roofline, other_kernel=other)
    else:
        roofline = rate("monarch_tc_kernel", f"monarch_tc_kernel<{wl.d}> (both stages, one persistent launch)",
                        0, wl.flops, wl.io_bytes)

    # end to end through the host-buffer entry point: H2D of Q, K, V, the call, D2H of out,
    # with the copies overlapped with the computation over chunks of batch-heads
    e2e = None
    if not args.no_e2e and grad:
        # per call the host sends Q, K, V, dO and reads dQ, dK, dV back
        d_q, d_k, d_v, d_do = (torch.empty_like(q0, device=device) for _ in range(4))
        hq, hk, hv = (x.pin_memory() for x in (q0, k0, v0))
        hdo = workloads.generate_upstream(wl).pin_memory()
        hdq, hdk, hdv = (torch.empty_like(q0).pin_memory() for _ in range(3))
        dq_b, dk_b, dv_b = (torch.empty_like(q0, device=device) for _ in range(3))
        ws_b = binding.monarch_attn_bwd_workspace(d_q, wl.T, wl.H, wl.W)

        def e2e_call():
            for h, d_ in ((hq, d_q), (hk, d_k), (hv, d_v), (hdo, d_do)):
                d_.copy_(h, non_blocking=True)
            binding.monarch_attn_bwd(d_q, d_k, d_v, d_do, wl.T, wl.H, wl.W, wl.fact, wl.tile_h, wl.tile_w,
                                     out=(dq_b, dk_b, dv_b), workspace=ws_b)
            for d_, h in ((dq_b, hdq), (dk_b, hdk), (dv_b, hdv)):
                h.copy_(d_, non_blocking=True)

        e2e_call()
        e2e_steps = max(1, min(args.steps, args.e2e_steps))
        barrier(device)
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_call()
        e1.record(stream)
        torch.cuda.synchronize(device)
        e2e_s = max_over_ranks(e0.elapsed_time(e1) / 1e3, device)
        e2e_val, e2e_ms = aggregate(world, wl.flops, e2e_steps, e2e_s)
        nbytes = q0.numel() * q0.element_size()
        e2e = {"value": e2e_val, "unit": "TFLOP/s", "ms_per_step": e2e_ms, "steps": e2e_steps,
               "h2d_bytes_per_step": 4 * nbytes, "d2h_bytes_per_step": 3 * nbytes,
               "api": "monarch_attn_bwd with pinned host copies of Q, K, V, dO in and dQ, dK, dV out"}
    elif not args.no_e2e and chunk:
        # per chunk the host sends the new frames' Q, K, V and reads the output
        # back; the context and y1_new stay on the device (the cache of an
        # autoregressive loop lives in HBM)
        hq, hk, hv = (x.pin_memory() for x in (q0, k0, v0))
        hout = torch.empty_like(q0).pin_memory()
        dq, dk, dv, dout, kc, yc, y1 = sets[0]

        def e2e_call():
            for h, d_ in ((hq, dq), (hk, dk), (hv, dv)):
                d_.copy_(h, non_blocking=True)
            binding.monarch_attn_fwd_chunk(dq, dk, dv, kc, yc, wl.T_ctx, wl.T, wl.H, wl.W, wl.fact,
                                           wl.tile_h, wl.tile_w, out=dout, y1_new=y1)
            hout.copy_(dout, non_blocking=True)

        for _ in range(2):
            e2e_call()
        e2e_steps = max(1, min(args.steps, args.e2e_steps))
        barrier(device)
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_call()
        e1.record(stream)
        torch.cuda.synchronize(device)
        e2e_s = max_over_ranks(e0.elapsed_time(e1) / 1e3, device)
        e2e_val, e2e_ms = aggregate(world, wl.flops, e2e_steps, e2e_s)
        nbytes = q0.numel() * q0.element_size()
        e2e = {"value": e2e_val, "unit": "TFLOP/s", "ms_per_step": e2e_ms, "steps": e2e_steps,
               "h2d_bytes_per_step": 3 * nbytes, "d2h_bytes_per_step": nbytes,
               "api": "monarch_attn_fwd_chunk with pinned host copies of Q, K, V in and out back "
                      "(context resident on the device)"}
    elif not args.no_e2e:
        hq, hk, hv = (x.pin_memory() for x in (q0, k0, v0))
        hout = torch.empty_like(q0).pin_memory()
        dq, dk, dv, dout = sets[0]
        def e2e_call():
            binding.monarch_attn_fwd_host_pipelined(hq, hk, hv, hout, dq, dk, dv, dout, wl.T, wl.H, wl.W,
                                                    wl.fact, wl.tile_h, wl.tile_w, nchunks=args.e2e_chunks)

        for _ in range(2):
            e2e_call()
        e2e_steps = max(1, min(args.steps, args.e2e_steps))
        barrier(device)
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_call()
        e1.record(stream)
        torch.cuda.synchronize(device)
        e2e_s = max_over_ranks(e0.elapsed_time(e1) / 1e3, device)
        e2e_val, e2e_ms = aggregate(world, wl.flops, e2e_steps, e2e_s)
        nbytes = q0.numel() * q0.element_size()
        e2e = {"value": e2e_val, "unit": "TFLOP/s", "ms_per_step": e2e_ms, "steps": e2e_steps,
               "h2d_bytes_per_step": 3 * nbytes, "d2h_bytes_per_step": nbytes,
               "api": f"monarch_attn_fwd_host_pipelined ({args.e2e_chunks} chunks of batch-heads)"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        try:
            import oracle
            oracle.build()
            if chunk or row or grad:
                sampler = oracle_chunk_sample if chunk else (oracle_bwd_sample if grad else oracle_head_sample)
                val, dt, reps = sampler(wl, args.cpu_seconds)
                what = "chunk" if chunk else ("fp64 gradients" if grad else "full forward")
                sample = f"{reps} head(s) of the {what} ({dt:.1f} s)"
            else:
                qs, ks, vs, groups, fpg = oracle_sample(wl, args.cpu_seconds)
                val, dt = time_oracle(wl, qs, ks, vs, groups, fpg)
                sample = (f"{len(groups)} stage-2 groups x {wl.T} rows of one head "
                          f"({len(groups) * fpg / 1e9:.2f} GFLOP, {dt:.1f} s)")
            cpu = {"value": val, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
                   "sample": sample}
        except Exception as exc:  # the CPU baseline is a report, not the product
            cpu = {"value": None, "unit": "TFLOP/s", "cores": None, "kind": "oracle",
                   "sample": f"failed: {exc}"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": wl.dtype, "data": "synthetic",
            "config": workload_config(wl, {
                "parallelism": f"replicas x{world} (independent (batch, head) problems; no collective)",
                "l2": ("inputs larger than L2: 3 rotating buffer sets of Q, K, V, out, context K and Y1, "
                       "y1_new" if chunk else
                       "inputs larger than L2: 3 rotating buffer sets of Q, K, V, out (1.2 GB)")}),
            "pct_of_bf16_peak": {"measured_burst": value / world / peak,
                                 "measured_sustained": value / world / peak_sus,
                                 "datasheet_2250": value / world / 2250.0},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "warm_l2": warm,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--soak-seconds", type=float, default=2.0)
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-chunks", type=int, default=6,
                    help="batch-head chunks the end-to-end call pipelines its copies over")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--warm-steps", type=int, default=20,
                    help="calls timed on one reused buffer set (warm L2), reported as warm_l2; 0 skips")
    ap.add_argument("--clock-log", default=None,
                    help="directory for the raw nvidia-smi clock samples (default: a temporary file)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--traffic", type=float, default=None,
                    help="dram bytes per launch of the dominant kernel from an ncu capture "
                         "(default: the committed profile summary, if the kernel is unchanged)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
