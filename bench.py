"""Throughput of exact attention (forward + backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]
    python bench.py --sweep [--sweep-points NAME,...]

A step is one forward and one backward pass (every stage of the path) over one
batch of the long-context workload, B=1, H=32, N=16384, d=128, causal, bf16
(seeded synthetic N(0,1) inputs; Q, K, V and dO are 128 MiB each, so every
step's inputs are larger than the 126 MB L2).  Throughput is algorithmic
TFLOP/s: 4*d flops per unmasked (query, key) pair for the forward, 10*d for the
backward (five matmuls, one of them the recomputation of Q K^T).

With N > 1 (launched by torch.distributed.run, one rank per GPU) every rank
processes its own batch of that workload (weak scaling; no collective on the
data path), and the reported time is the maximum over ranks.

Rank 0 prints one JSON line.  ``--impl reference`` times the fp64 CPU oracle on
the host cores instead (a bounded sample of the same workload per step).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
METRIC = "attention fwd/bwd TFLOP/s (bf16, d=128, N 1k-32k) and % of B200 BF16 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_bwd_dkdv_long_context_traffic.txt")
KERNEL_SOURCES = [os.path.join(ROOT, "exact_attention_106_b200", "csrc", f) for f in ("bwd.cuh", "ptx.cuh")]


# --------------------------------------------------------------------- utils
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    """Hash of the kernel sources' code: comments and whitespace are left out,
    so that a change to them keeps a recorded measurement valid."""
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(p, encoding="utf-8") as f:
            code = f.read()
        code = re.sub(r"/\*.*?\*/", " ", code, flags=re.S)
        code = re.sub(r"//[^\n]*", " ", code)
        h.update(" ".join(code.split()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload):
    """Per-launch DRAM bytes of the backward main kernel from the committed ncu
    summary, or None if absent, taken on another workload or on a different
    kernel source."""
    try:
        kv = {}
        with open(TRAFFIC_FILE) as f:
            for line in f:
                if ":" in line and not line.lstrip().startswith("#"):
                    a, b = line.split(":", 1)
                    kv[a.strip()] = b.strip()
        if kv.get("kernel_source_sha256_16") != kernel_source_hash() or kv.get("workload") != workload:
            return None
        return float(kv["traffic_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.out = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.gpu_index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        if not self.out:
            return None
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


def reduce_max(value: float, device) -> float:
    """Maximum of a per-rank scalar over all ranks (identity without a process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, flops_per_step: float, steps: int, max_ms: float) -> float:
    """Whole-job TFLOP/s: every rank processes `steps` steps of its own batch;
    the time is the slowest rank's."""
    return world * flops_per_step * steps / (max_ms * 1e-3) / 1e12


def rank_workload(base, rank: int):
    """Each rank gets its own batch: same shape, seeds shifted by the rank."""
    import dataclasses
    return dataclasses.replace(base, seed_base=base.seed_base + 10 * rank)


# -------------------------------------------------------------- CPU baseline
def oracle_sample(w, rows: int):
    """The first `rows` tokens of head (0, 0) of workload w: under the causal
    mask this is itself a complete attention problem of length `rows`."""
    from exact_attention_106_b200 import workloads as W
    import dataclasses
    sub = dataclasses.replace(w, B=1, H=1, N=rows)
    q, k, v, do = W.make_inputs(sub)
    return sub, q, k, v, do


def time_oracle(w, rows: int):
    import oracle
    sub, q, k, v, do = oracle_sample(w, rows)
    t0 = time.perf_counter()
    oracle.backward(q, k, v, do, sub.softmax_scale, sub.causal)
    dt = time.perf_counter() - t0
    return (sub.fwd_flops() + sub.bwd_flops()) / dt / 1e12, dt, sub


def time_oracle_heads(w, heads: int):
    """fwd + bwd of the first `heads` full heads of batch 0 of workload w."""
    import dataclasses
    import oracle
    from exact_attention_106_b200 import workloads as W
    q, k, v, do = W.make_inputs(w)
    sel = [(0, h) for h in range(heads)]
    t0 = time.perf_counter()
    oracle.backward(q[:1, :heads], k[:1, :heads], v[:1, :heads], do[:1, :heads], w.softmax_scale, w.causal)
    dt = time.perf_counter() - t0
    sub = dataclasses.replace(w, B=1, H=heads)
    return (sub.fwd_flops() + sub.bwd_flops()) / dt / 1e12, dt, len(sel)


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


# ------------------------------------------------------------------ our arm
def run_ours(args, rank, world, local_rank):
    import exact_attention_106_b200 as ex
    from exact_attention_106_b200 import workloads as W

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = rank_workload(W.by_name(args.workload), rank)
    B, H, N, d = w.shape
    q, k, v, do = W.make_inputs(w)
    torch.cuda.reset_peak_memory_stats(dev)
    qd, kd, vd, dod = (x.to(dev) for x in (q, k, v, do))
    o = torch.empty_like(qd)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty_like(qd) for _ in range(3))
    ws = ex.alloc_workspace(B, H, N, d, dev)
    stream = torch.cuda.current_stream(dev)

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        ex.forward(qd, kd, vd, causal=w.causal, scale=w.softmax_scale, out=o, lse=lse)
        if evs:
            evs[1].record(stream)
        for i, _ in enumerate(ex.bwd_stages(qd, kd, vd, o, lse, dod, dq, dk, dv, ws, causal=w.causal,
                                            scale=w.softmax_scale)):
            if evs:
                evs[2 + i].record(stream)

    import torch.distributed as dist
    dist_on = dist.is_available() and dist.is_initialized()

    def barrier():
        if dist_on:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        step()
    if ex.device_status(dev) != 0:
        raise RuntimeError("device status not clean after warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    with ClockSampler(local_rank) as clk:
        t_start.record(stream)
        for s in range(args.steps):
            step(evs[s])
        t_end.record(stream)
        barrier()
    elapsed_ms = t_start.elapsed_time(t_end)
    peak_alloc = torch.cuda.max_memory_allocated(dev)  # inputs, outputs, workspace: linear in N
    status = ex.device_status(dev)
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")
    per_kernel = {name: [evs[s][i].elapsed_time(evs[s][i + 1]) for s in range(args.steps)]
                  for i, name in enumerate(["fwd", "bwd_preprocess", "bwd_dkdv", "bwd_dq_convert"])}
    max_ms = reduce_max(elapsed_ms, dev)
    flops_step = w.fwd_flops() + w.bwd_flops()

    # e2e: one C-ABI call per step on page-locked host buffers (attn_fwd_bwd_host:
    # inputs copied in, fwd + bwd, results copied out, pipelined over head chunks)
    hq, hk, hv, hdo = (x.pin_memory() for x in (q, k, v, do))
    ho, hdq, hdk, hdv = (torch.empty(w.shape, dtype=torch.bfloat16).pin_memory() for _ in range(4))
    hlse = torch.empty((B, H, N), dtype=torch.float32).pin_memory()
    del qd, kd, vd, dod, o, lse, dq, dk, dv, ws
    torch.cuda.empty_cache()
    hbuf = torch.empty(max(1, ex.host_buffer_bytes(B, H, N, d)), dtype=torch.uint8, device=dev)

    def e2e_step():
        ex.forward_backward_host(hq, hk, hv, hdo, (ho, hlse, hdq, hdk, hdv), causal=w.causal,
                                 scale=w.softmax_scale, device=dev, dev_buffer=hbuf)

    e2e_steps = max(1, min(args.steps, 20))
    for _ in range(2):
        e2e_step()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    barrier()
    e2e_ms = reduce_max(e0.elapsed_time(e1), dev)
    if ex.device_status(dev) != 0:
        raise RuntimeError("device status not clean after the end-to-end steps")
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hdo))
    d2h = sum(x.numel() * x.element_size() for x in (ho, hlse, hdq, hdk, hdv))

    if rank != 0:
        return None
    peaks, peak_src = load_peaks()
    mean = {k_: statistics.mean(v_) for k_, v_ in per_kernel.items()}
    fwd_tf = w.fwd_flops() / (mean["fwd"] * 1e-3) / 1e12
    bwd_ms = mean["bwd_preprocess"] + mean["bwd_dkdv"] + mean["bwd_dq_convert"]
    bwd_tf = w.bwd_flops() / (bwd_ms * 1e-3) / 1e12
    dkdv_tf = w.bwd_flops() / (mean["bwd_dkdv"] * 1e-3) / 1e12
    dominant = "bwd_dkdv" if mean["bwd_dkdv"] >= mean["fwd"] else "fwd"
    dom_tf = dkdv_tf if dominant == "bwd_dkdv" else fwd_tf
    # The timed region is a fraction of a second to a few seconds of
    # back-to-back launches: the burst peak is the denominator; the
    # sustained one (seconds under the power cap) is reported beside it.
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    value = job_throughput(world, flops_step, args.steps, max_ms)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        v_cpu, dt_cpu, nh = time_oracle_heads(w, args.cpu_heads)
        cpu = {"value": v_cpu, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
               "seconds": dt_cpu,
               "sample": f"fp64 numpy oracle, fwd+bwd of heads 0..{nh - 1} of batch 0 of {w.name} "
                         f"(full length {N}); algorithmic flops of those heads / time"}
    spec_peak = 2250.0
    tensor_mib = B * H * N * d * 2 / 2**20
    result = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "B": B, "H": H, "N": N, "d": d, "causal": w.causal,
                   "step": "forward + backward (all stages)", "parallelism": f"replicas x{world}",
                   "l2": (f"inputs larger than L2 (Q, K, V, dO {tensor_mib:.0f} MiB each per step)"
                          if 4 * tensor_mib > 126 else "inputs smaller than L2 (not flushed)")},
        "fwd_tflops": fwd_tf, "bwd_tflops": bwd_tf,
        "pct_of_peak": {"fwd_of_burst": fwd_tf / peak, "bwd_of_burst": bwd_tf / peak,
                        "fwd_of_sustained": fwd_tf / peak_sus, "bwd_of_sustained": bwd_tf / peak_sus,
                        "fwd_of_spec_2250": fwd_tf / spec_peak, "bwd_of_spec_2250": bwd_tf / spec_peak,
                        "peak_source": peak_src},
        "kernels": {k_: {"mean_ms": mean[k_]} for k_ in mean},
        "roofline": {"kernel": "attn_bwd_kernel<128, bf16, 0>" if dominant == "bwd_dkdv" else "attn_fwd_kernel<128, bf16, 0>",
                     "bound": "tensor", "achieved": dom_tf, "peak": peak, "unit": "TFLOP/s",
                     "frac": dom_tf / peak, "peak_kind": f"bf16 burst ({peak_src})",
                     "frac_of_sustained": dom_tf / peak_sus,
                     "traffic": recorded_traffic(w.name) if dominant == "bwd_dkdv" else None},
        "cpu_baseline": cpu,
        "e2e": {"value": job_throughput(world, flops_step, e2e_steps, e2e_ms), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "memory": {"peak_allocated_bytes": peak_alloc, "one_bf16_score_matrix_bytes": B * H * N * N * 2},
        "clocks": clk.summary(),
        "gpu_launches": 4 * args.steps,
    }
    result["kernels"]["fwd"]["tflops"] = fwd_tf
    result["kernels"]["bwd_dkdv"]["tflops"] = dkdv_tf
    return result


# ------------------------------------------------------------------ sweep
SPEC_PEAK_TFLOPS = 2250.0  # dense bf16, B200 spec
SM_COUNT = 148
FLOP_PER_SM_CYCLE = 8192   # bf16 MMA rate of one SM (128x128x16 per 64 cycles)


def sweep_workloads():
    from exact_attention_106_b200 import workloads as W
    return W.sweep() + [W.SINGLE_HEAD_32K, W.SINGLE_HEAD_32K_CAUSAL]


def time_point(w, dev, min_reps: int, min_seconds: float, flush):
    """Median and minimum CUDA-event time of the forward and of each backward
    stage on workload w, with the L2 flushed (256 MiB write) before each
    forward + backward repetition; repetitions are raised until the timed launches of the point last
    at least `min_seconds`, so the clock samples cover them."""
    import exact_attention_106_b200 as ex
    from exact_attention_106_b200 import workloads as W
    B, H, N, d = w.shape
    q, k, v, do = (x.to(dev) for x in W.make_inputs(w))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    ws = ex.alloc_workspace(B, H, N, d, dev)
    stream = torch.cuda.current_stream(dev)
    names = ["fwd", "bwd_preprocess", "bwd_dkdv", "bwd_dq_convert"]

    def rep():
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(8)]
        flush.zero_()
        evs[0].record(stream)
        ex.forward(q, k, v, causal=w.causal, scale=w.softmax_scale, out=o, lse=lse)
        evs[1].record(stream)
        gen = ex.bwd_stages(q, k, v, o, lse, do, dq, dk, dv, ws, causal=w.causal, scale=w.softmax_scale)
        for i in range(3):
            evs[2 + 2 * i].record(stream)
            next(gen)
            evs[3 + 2 * i].record(stream)
        return evs

    for _ in range(3):
        rep()
    torch.cuda.synchronize(dev)
    t0 = time.perf_counter()
    evs = [rep()]
    torch.cuda.synchronize(dev)
    est = max(time.perf_counter() - t0, 1e-4)
    reps = max(min_reps, int(min_seconds / est) + 1)
    with ClockSampler(dev.index or 0) as clk:
        evs = [rep() for _ in range(reps)]
        torch.cuda.synchronize(dev)
    if ex.device_status(dev) != 0:
        raise RuntimeError(f"device status not clean after {w.name}")
    ms = {n: sorted(e[2 * i].elapsed_time(e[2 * i + 1]) for e in evs) for i, n in enumerate(names)}
    return {n: {"median_ms": statistics.median(v), "min_ms": v[0]} for n, v in ms.items()}, reps, clk.summary()


def run_sweep(args):
    """One JSON line per point of the sweep (fixed 16384 tokens per batch,
    N in 512..16384, d in {64, 128}, causal and not) and of the single-head
    N = 32768 d = 128 problems: forward and backward TFLOP/s and their
    fractions of the burst, spec and clock-scaled tensor peaks."""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    only = set(args.sweep_points.split(",")) if args.sweep_points else None
    rows = []
    for w in sweep_workloads():
        if only and w.name not in only:
            continue
        t, reps, clk = time_point(w, dev, args.sweep_reps, args.sweep_seconds, flush)
        fwd_ms = t["fwd"]["median_ms"]
        bwd_ms = t["bwd_preprocess"]["median_ms"] + t["bwd_dkdv"]["median_ms"] + t["bwd_dq_convert"]["median_ms"]
        fwd_tf = w.fwd_flops() / (fwd_ms * 1e-3) / 1e12
        bwd_tf = w.bwd_flops() / (bwd_ms * 1e-3) / 1e12
        mhz = clk["sm_mhz"] if clk else None
        clock_peak = SM_COUNT * FLOP_PER_SM_CYCLE * mhz * 1e6 / 1e12 if mhz else None
        row = {"point": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal, "reps": reps,
               "fwd_ms": fwd_ms, "bwd_ms": bwd_ms, "stages_ms": t,
               "fwd_tflops": fwd_tf, "bwd_tflops": bwd_tf,
               "fwd_of_burst": fwd_tf / burst, "bwd_of_burst": bwd_tf / burst,
               "fwd_of_spec_2250": fwd_tf / SPEC_PEAK_TFLOPS, "bwd_of_spec_2250": bwd_tf / SPEC_PEAK_TFLOPS,
               "fwd_of_clock_peak": fwd_tf / clock_peak if clock_peak else None,
               "bwd_of_clock_peak": bwd_tf / clock_peak if clock_peak else None,
               "burst_peak": burst, "peak_source": peak_src, "clocks": clk}
        rows.append(row)
        print(json.dumps(row), flush=True)
    for row in (kvsplit_points(dev, flush, burst, peak_src, args, only) + fp8_points(dev, flush, burst, args, only)
                + hdim256_points(dev, flush, burst, args, only) + fp16_points(dev, flush, burst, args, only)):
        rows.append(row)
        print(json.dumps(row), flush=True)
    return rows


def fp16_points(dev, flush, burst, args, only):
    """The long-context workload on fp16 tensors (attn_fwd_fp16 / attn_bwd_fp16),
    forward and whole backward."""
    import exact_attention_106_b200 as ex
    from exact_attention_106_b200 import workloads as W
    w = W.LONG_CONTEXT
    name = w.name + "_fp16"
    if only and name not in only:
        return []
    q, k, v, do = (x.to(dev) for x in W.make_inputs(w, dtype=torch.float16))
    o = torch.empty_like(q)
    lse = torch.empty(w.shape[:3], dtype=torch.float32, device=dev)
    grads = tuple(torch.empty_like(q) for _ in range(3))
    ws = ex.alloc_workspace(*w.shape, dev)
    fwd = lambda: ex.forward(q, k, v, causal=True, scale=w.softmax_scale, out=o, lse=lse)  # noqa: E731
    fwd()
    bwd = lambda: ex.backward(q, k, v, o, lse, do, causal=True, scale=w.softmax_scale, workspace=ws,  # noqa: E731
                              out=grads)
    f_med, _, reps, clk = time_fn(fwd, dev, flush, args.sweep_reps, args.sweep_seconds)
    b_med, _, _, _ = time_fn(bwd, dev, flush, args.sweep_reps, args.sweep_seconds)
    ftf = w.fwd_flops() / (f_med * 1e-3) / 1e12
    btf = w.bwd_flops() / (b_med * 1e-3) / 1e12
    return [{"point": name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": True, "reps": reps,
             "fwd_ms": f_med, "fwd_tflops": ftf, "bwd_ms_all_stages": b_med, "bwd_tflops_all_stages": btf,
             "fwd_of_burst": ftf / burst, "bwd_of_burst": btf / burst, "clocks": clk}]


def hdim256_points(dev, flush, burst, args, only):
    """The forward at head_dim 256 (one 128-row sub-tile per CTA)."""
    import exact_attention_106_b200 as ex
    from exact_attention_106_b200 import workloads as W
    out = []
    for w in W.HDIM256:
        if only and w.name not in only:
            continue
        q, k, v, _ = (x.to(dev) if x is not None else None for x in W.make_inputs(w, with_grad_out=False))
        o = torch.empty_like(q)
        lse = torch.empty(w.shape[:3], dtype=torch.float32, device=dev)
        med, mn, reps, clk = time_fn(lambda: ex.forward(q, k, v, causal=w.causal, scale=w.softmax_scale, out=o,
                                                       lse=lse), dev, flush, args.sweep_reps, args.sweep_seconds)
        tf = w.fwd_flops() / (med * 1e-3) / 1e12
        mhz = clk["sm_mhz"] if clk else None
        out.append({"point": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal, "reps": reps,
                    "fwd_ms": med, "fwd_min_ms": mn, "fwd_tflops": tf, "fwd_of_burst": tf / burst,
                    "fwd_of_spec_2250": tf / SPEC_PEAK_TFLOPS,
                    "fwd_of_clock_peak": tf / (SM_COUNT * FLOP_PER_SM_CYCLE * mhz * 1e-6) if mhz else None,
                    "clocks": clk})
        del q, k, v, o, lse
        torch.cuda.empty_cache()
    return out


def fp8_points(dev, flush, burst, args, only):
    """The e4m3 forward (attn_fwd_fp8) on the d = 128 sweep shapes, causal and
    not.  Its tensor-core peak is twice the bf16 one (the nominal ratio of
    the dense e4m3 and bf16 rates, 4.5 / 2.25 PFLOP/s), applied to the
    measured bf16 burst peak."""
    import exact_attention_106_b200 as ex
    from exact_attention_106_b200 import workloads as W
    out = []
    for w in [x for x in W.sweep() if x.d == 128 and x.N >= 4096] + [W.LONG_CONTEXT]:
        name = w.name + "_fp8"
        if only and name not in only:
            continue
        q, k, v, _ = W.make_inputs(w, with_grad_out=False, dtype=torch.float32)
        sc = [float(t.abs().max()) / 448.0 for t in (q, k, v)]
        q8, k8, v8 = ((t / s).to(torch.float8_e4m3fn).to(dev) for t, s in zip((q, k, v), sc))
        del q, k, v
        o = torch.empty(w.shape, dtype=torch.bfloat16, device=dev)
        lse = torch.empty(w.shape[:3], dtype=torch.float32, device=dev)
        med, mn, reps, clk = time_fn(lambda: ex.forward_fp8(q8, k8, v8, *sc, causal=w.causal, scale=w.softmax_scale,
                                                           out=o, lse=lse), dev, flush, args.sweep_reps,
                                     args.sweep_seconds)
        tf = w.fwd_flops() / (med * 1e-3) / 1e12
        mhz = clk["sm_mhz"] if clk else None
        out.append({"point": name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal, "reps": reps,
                    "fwd_ms": med, "fwd_min_ms": mn, "fwd_tflops": tf, "fp8_peak": 2 * burst,
                    "fwd_of_fp8_peak": tf / (2 * burst), "fwd_of_fp8_spec_4500": tf / 4500.0,
                    "fwd_of_fp8_clock_peak": tf / (2 * SM_COUNT * FLOP_PER_SM_CYCLE * mhz * 1e-6) if mhz else None,
                    "clocks": clk})
        del q8, k8, v8, o, lse
        torch.cuda.empty_cache()
    return out


def time_fn_block(fn, dev, min_reps: int, min_seconds: float):
    """For inputs far larger than L2 (no flush needed): calls timed back to
    back in blocks of 10 with one event pair per block, so that the host's
    launch latency overlaps the previous call; (median, min) per call over
    the blocks, and the clocks sampled meanwhile."""
    stream = torch.cuda.current_stream(dev)
    for _ in range(3):
        fn()
    torch.cuda.synchronize(dev)
    t0 = time.perf_counter()
    for _ in range(10):
        fn()
    torch.cuda.synchronize(dev)
    blocks = max(min_reps, int(min_seconds / max(time.perf_counter() - t0, 1e-4)) + 1)
    evs = []
    with ClockSampler(dev.index or 0) as clk:
        for _ in range(blocks):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(10):
                fn()
            b.record(stream)
            evs.append((a, b))
        torch.cuda.synchronize(dev)
    ms = sorted(a.elapsed_time(b) / 10 for a, b in evs)
    return statistics.median(ms), ms[0], 10 * blocks, clk.summary()


def time_fn(fn, dev, flush, min_reps: int, min_seconds: float):
    """Median / min CUDA-event time of fn() with the L2 flushed before each
    call, and the clocks sampled while the timed calls run."""
    stream = torch.cuda.current_stream(dev)
    for _ in range(3):
        fn()
    torch.cuda.synchronize(dev)
    t0 = time.perf_counter()
    fn()
    torch.cuda.synchronize(dev)
    reps = max(min_reps, int(min_seconds / max(time.perf_counter() - t0, 1e-4)) + 1)
    evs = []
    with ClockSampler(dev.index or 0) as clk:
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            flush.zero_()
            a.record(stream)
            fn()
            b.record(stream)
            evs.append((a, b))
        torch.cuda.synchronize(dev)
    ms = sorted(a.elapsed_time(b) for a, b in evs)
    return statistics.median(ms), ms[0], reps, clk.summary()


def kvsplit_points(dev, flush, burst, peak_src, args, only):
    """The split-key forward (attn_fwd_kvsplit): the single-head 32K causal
    problem (L2 flushed before each call), and the decode workloads
    (bandwidth-bound: GB/s of algorithmic HBM bytes against the HBM peak;
    their 4.3 GB of K and V exceed L2, so calls run back to back)."""
    import exact_attention_106_b200 as ex
    from exact_attention_106_b200 import workloads as W
    peaks, _ = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    out = []
    w = W.SINGLE_HEAD_32K_CAUSAL
    name = w.name + "_kvsplit"
    if not only or name in only:
        q, k, v, _ = (x.to(dev) if x is not None else None for x in W.make_inputs(w, with_grad_out=False))
        splits, need = ex.kvsplit_plan(w.B, w.H, w.N, w.N, w.d, True, 0)
        ws = torch.empty(max(1, need), dtype=torch.uint8, device=dev)
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
        med, mn, reps, clk = time_fn(lambda: ex.forward_kvsplit(q, k, v, causal=True, scale=w.softmax_scale,
                                                               workspace=ws, out=o, lse=lse), dev, flush,
                                     args.sweep_reps, args.sweep_seconds)
        tf = w.fwd_flops() / (med * 1e-3) / 1e12
        mhz = clk["sm_mhz"] if clk else None
        out.append({"point": name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": True, "splits": splits,
                    "reps": reps, "fwd_ms": med, "fwd_min_ms": mn, "fwd_tflops": tf, "fwd_of_burst": tf / burst,
                    "fwd_of_spec_2250": tf / SPEC_PEAK_TFLOPS,
                    "fwd_of_clock_peak": tf / (SM_COUNT * FLOP_PER_SM_CYCLE * mhz * 1e-6) if mhz else None,
                    "burst_peak": burst, "peak_source": peak_src, "clocks": clk})
    for w in W.DECODES:
        if only and w.name not in only:
            continue
        q, k, v = (x.to(dev) for x in W.make_decode_inputs(w))
        splits, need = ex.kvsplit_plan(w.B, w.H, w.Nq, w.Nk, w.d, w.causal, 0)
        ws = torch.empty(max(1, need), dtype=torch.uint8, device=dev)
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=dev)
        # K and V are 4.3 GB, far beyond L2: no flush, calls back to back
        med, mn, reps, clk = time_fn_block(lambda: ex.forward_kvsplit(q, k, v, causal=w.causal,
                                                                     scale=w.softmax_scale, workspace=ws, out=o,
                                                                     lse=lse), dev, args.sweep_reps,
                                           args.sweep_seconds)
        gbs = w.bytes_moved() / (med * 1e-3) / 1e9
        out.append({"point": w.name, "B": w.B, "H": w.H, "Nq": w.Nq, "Nk": w.Nk, "d": w.d, "causal": w.causal,
                    "splits": splits, "reps": reps, "fwd_ms": med, "fwd_min_ms": mn,
                    "fwd_tflops": w.fwd_flops() / (med * 1e-3) / 1e12, "bytes": w.bytes_moved(),
                    "workspace_bytes": need, "gbs": gbs, "hbm_peak_gbs": hbm, "frac_of_hbm": gbs / hbm,
                    "clocks": clk})
        del q, k, v, ws, o, lse
        torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------ reference arm
def run_reference(args, rank):
    from exact_attention_106_b200 import workloads as W
    if rank != 0:
        return None
    w = W.by_name(args.workload)
    rows = args.ref_rows
    vals = []
    for _ in range(args.warmup):
        time_oracle(w, rows)
    t_total = 0.0
    for _ in range(args.steps):
        v_, dt, sub = time_oracle(w, rows)
        vals.append(v_)
        t_total += dt
    value = args.steps * (sub.fwd_flops() + sub.bwd_flops()) / t_total / 1e12
    cores = blas_threads()
    sample = (f"fp64 numpy oracle, fwd+bwd of the first {rows} tokens of head (0,0) of {w.name} "
              f"(a complete causal problem 1x1x{rows}x{w.d}) per step")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
                   "step": "forward + backward", "sample_rows": rows},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="long_context_1x32x16384x128_causal")
    ap.add_argument("--cpu-heads", type=int, default=3, help="full heads timed for cpu_baseline")
    ap.add_argument("--ref-rows", type=int, default=2048, help="oracle sample size per reference step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", action="store_true",
                    help="time every sweep point and the single-head 32K problems (one JSON line each)")
    ap.add_argument("--sweep-points", default="", help="comma-separated subset of sweep point names")
    ap.add_argument("--sweep-reps", type=int, default=10, help="minimum timed repetitions per point")
    ap.add_argument("--sweep-seconds", type=float, default=0.5, help="minimum timed seconds per point")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}")

    if args.sweep:
        if world != 1 or args.impl != "ours":
            ap.error("--sweep runs on one GPU, our implementation")
        run_sweep(args)
        return 0
    if args.impl == "reference":
        out = run_reference(args, rank)
    else:
        if world > 1:
            import datetime
            import torch.distributed as dist
            torch.cuda.set_device(local_rank)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local_rank))
        try:
            out = run_ours(args, rank, world, local_rank)
        finally:
            import torch.distributed as dist
            if dist.is_available() and dist.is_initialized():
                dist.destroy_process_group()
    if out is not None:
        print(json.dumps(out), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
