#!/usr/bin/env python
"""Benchmark of the attention core: global attention over S=100 frames x 1031
tokens (103,100 tokens, 16 heads x 64, bf16), the headline workload.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one vggt_attn_global call (QK-LayerNorm + RoPE prologue, then the
tcgen05 attention core) on inputs resident in HBM.  `value` is the
algorithmic TFLOP/s (4 * N^2 * 64 * H per call: QK^T and PV only) summed over
all ranks, from CUDA-event time (max over ranks).  Side measurements in the
same run: `e2e` (the same steps from pinned host buffers, H2D + D2H inside the
timed region), `roofline` (the core kernel alone against the measured bf16
peak), `modes` (ms per mode on the other workloads), `clocks` (nvidia-smi
sampled during the timed region) and `cpu_baseline` (the fp64 oracle on a
bounded sample, on this host's cores).

Multi-GPU: one process per GPU (torchrun); every rank runs its own,
independent copy of the workload (an independent scene), so per-GPU work is
fixed and no data crosses ranks ("scaling": "weak").  `--impl reference` runs
the fp64 oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

HEADLINE = 3                      # global, S=100, 103,100 tokens, H=16
METRIC = "global-attn TFLOP/s & % bf16 tensor peak (S=100, 103k tok); ms/layer per mode"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
CORE_SRC = os.path.join(ROOT, "vit_attention_b200", "csrc", "attention_sm100.cuh")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_core_global_S100_traffic.txt")


def attention_flops(mode: str, shape) -> float:
    """Algorithmic flops of one call: 4 * Nq * Nk * 64 per head (QK^T + PV)."""
    if mode == "global":
        n = shape.S * shape.T
        return 4.0 * n * n * 64 * shape.H
    if mode == "frame":
        return 4.0 * shape.S * shape.T * shape.T * 64 * shape.H
    n = shape.S * shape.n_special
    return 4.0 * n * n * 64 * shape.H


def io_bytes(mode: str, shape) -> float:
    """Minimum HBM bytes of one call: read the q/k/v it uses, write its output rows."""
    rows = shape.S * (shape.n_special if mode == "register" else shape.T)
    return rows * shape.H * 64 * 2 * 4.0


# ---------------------------------------------------------------- distributed plumbing
def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), \
        int(os.environ.get("LOCAL_RANK", "0"))


def shard_plan(world: int, rank: int, base_seed: int):
    """Weak scaling: rank r runs one independent copy of the workload (its own seed)."""
    return {"rank": rank, "world": world, "seed": base_seed + 7919 * rank, "problems": 1}


def scene_frames(S: int, world: int, rank: int) -> range:
    """Query-sharded global attention: rank r holds frames [r * S / world, (r + 1) * S / world) of the scene
    (consecutive blocks in rank order, the order the all-gather concatenates the ranks' keys in)."""
    if S % world:
        raise ValueError(f"--sharded splits the {S} frames evenly: {world} ranks do not divide them")
    per = S // world
    return range(rank * per, (rank + 1) * per)


def reduce_max(value: float, device=None) -> float:
    """Max of a scalar over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap", "utilization.gpu"]

    def __init__(self, device_index: int):
        self.proc = None
        self.lines = []
        self.gpu_id = None
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.gpu_id = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.gpu_id = str(device_index)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        samples = []
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                samples.append({"sm": float(parts[0]), "max": float(parts[1]), "power": float(parts[2]),
                                "hw": parts[3], "hwt": parts[4], "swt": parts[5], "pcap": parts[6],
                                "util": float(parts[7])})
            except ValueError:
                continue
        if not samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [s for s in samples if s["util"] >= 50] or samples
        reasons = set()
        for s in loaded:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if s[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s["sm"] for s in loaded), "sm_max_mhz": max(s["max"] for s in loaded),
                "reasons": sorted(reasons), "samples": len(loaded),
                "power_w_max": max(s["power"] for s in loaded)}


# ---------------------------------------------------------------- helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def core_source_hash() -> str:
    with open(CORE_SRC, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic():
    """DRAM bytes per launch of the core kernel from the committed ncu summary,
    or None when absent or taken on a different kernel source."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    text = open(TRAFFIC_FILE).read()
    m_b = re.search(r"dram_bytes_per_launch\s*=\s*([0-9.eE+]+)", text)
    m_h = re.search(r"kernel_source_sha256_16\s*=\s*([0-9a-f]+)", text)
    if not m_b or not m_h or m_h.group(1) != core_source_hash():
        return None
    return float(m_b.group(1))


def device_inputs(x, device):
    import torch
    qkv = torch.from_numpy(x["qkv"].view(np.int16)).to(device).view(torch.bfloat16)
    prm = {k: torch.from_numpy(np.ascontiguousarray(x[k])).to(device)
           for k in ("q_gamma", "q_beta", "k_gamma", "k_beta")}
    return qkv, prm


def cuda_time_ms(fn, stream, iters: int) -> float:
    """Average ms per call of fn() over `iters` calls, CUDA events on `stream`."""
    import torch
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(iters):
        fn()
    end.record(stream)
    end.synchronize()
    return start.elapsed_time(end) / iters


# ---------------------------------------------------------------- oracle (CPU baseline / reference arm)
_ORACLE_INPUTS = {}


def oracle_sample(workload, n_queries: int, seed: int = 0):
    """Time the fp64 oracle on `n_queries` seeded queries of `workload` (global mode).

    The seeded inputs are drawn once and kept; the timed region is the oracle
    call alone (QK-LayerNorm + RoPE of every key and of the sampled queries,
    then their attention over all keys).
    Returns (seconds, algorithmic flops of the sample, threads used)."""
    import oracle as O
    from threadpoolctl import threadpool_info
    if workload.name not in _ORACLE_INPUTS:
        _ORACLE_INPUTS[workload.name] = W.make_inputs(workload)
    x = _ORACLE_INPUTS[workload.name]
    shape = workload.shape
    q = W.query_subset(shape.S * shape.T, n_queries, workload.seed + seed)
    t0 = time.perf_counter()
    O.attn_global(shape, x, q)
    dt = time.perf_counter() - t0
    n = shape.S * shape.T
    flops = 4.0 * n_queries * n * 64 * shape.H
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    return dt, flops, threads


def headline_config(w, world: int = 1):
    """The `config` of the JSON line; both arms (ours and --impl reference) print this same object."""
    shape = w.shape
    qkv_mb = shape.S * shape.T * 3 * shape.H * 64 * 2 / 1e6
    ws_mb = 2 * shape.S * shape.T * shape.H * 64 * 2 / 1e6
    return {"workload": w.name, "mode": "global", "frames": shape.S, "tokens": shape.S * shape.T,
            "heads": shape.H, "head_dim": 64, "flops_per_step_per_gpu": attention_flops("global", shape),
            "l2": f"no flush: qkv {qkv_mb:.0f} MB + workspace {ws_mb:.0f} MB read per step exceed the 126 MB L2",
            "parallelism": f"independent replicas x{world} (weak)"}


def cpu_baseline(n_queries: int):
    w = W.workload(HEADLINE)
    dt, flops, threads = oracle_sample(w, n_queries)
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"fp64 numpy oracle, global mode, {n_queries} seeded queries x all 16 heads over all "
                      f"{w.shape.S * w.shape.T} keys (incl. LN+RoPE of every key), {dt:.1f} s",
            "seconds": dt, "queries": n_queries}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    w = W.workload(HEADLINE)
    n_q = args.ref_queries
    times = []
    for i in range(args.warmup + args.steps):
        dt, flops, threads = oracle_sample(w, n_q, seed=i)
        if i >= args.warmup:
            times.append(dt)
    value = flops / statistics.mean(times) / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * statistics.mean(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": headline_config(w, world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": f"{n_q} seeded queries x 16 heads over all keys per step (QK-LayerNorm + "
                                       "RoPE of every key included), scaled by algorithmic flops"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- our arm
def run_ours(args):
    import torch
    import torch.distributed as dist
    import datetime

    import vit_attention_b200 as V

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    device = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)

    w = W.workload(args.workload)
    if w.modes != ("global",):
        raise SystemExit("--workload must name a global-mode workload")
    shape = w.shape
    plan = shard_plan(world, rank, w.seed)
    x = W.make_random_inputs(shape, plan["seed"], w.lowrank) if rank else W.make_inputs(w)
    qkv, prm = device_inputs(x, device)
    out = torch.empty((shape.S, shape.T, shape.H, 64), dtype=torch.bfloat16, device=device)
    ws_bytes = V.vggt_attn_workspace_size(shape, "global")
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=device)
    flops = attention_flops("global", shape)

    def step():
        V.vggt_attn_global(shape, qkv, prm["q_gamma"], prm["q_beta"], prm["k_gamma"], prm["k_beta"], out, ws,
                           ws_bytes, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    assert V.vggt_attn_read_status(ws, stream) == 0

    # ---- timed region: K steps, barrier + synchronize on both sides, max over ranks
    clocks = ClockSampler(device.index)
    clocks.start()
    time.sleep(0.4)
    barrier(device)
    torch.cuda.synchronize(device)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(args.steps):
        step()
    end.record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    clk = clocks.stop()
    ms_local = start.elapsed_time(end)
    ms = reduce_max(ms_local, device)
    status = V.vggt_attn_read_status(ws, stream)
    if status != 0:
        raise RuntimeError(f"device status {status} ({V.error_string(status)})")
    value = flops * args.steps * world / (ms / 1000.0) / 1e12
    launches = 2 * args.steps      # prologue + core per call

    # ---- roofline: the core kernel alone (CUDA events on its stream)
    peaks, peak_src = load_peaks()
    core_ms = cuda_time_ms(lambda: V.vggt_attn_core("global", shape, qkv, out, ws, ws_bytes, stream), stream,
                           max(3, args.steps))
    pro_ms = cuda_time_ms(lambda: V.vggt_attn_prologue("global", shape, qkv, prm["q_gamma"], prm["q_beta"],
                                                       prm["k_gamma"], prm["k_beta"], ws, ws_bytes, stream),
                          stream, 10)
    core_tflops = flops / (core_ms / 1000.0) / 1e12
    peak = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
    traffic = recorded_traffic()
    roofline = {"bound": "tensor", "achieved": core_tflops, "peak": peak, "unit": "TFLOP/s",
                "frac": core_tflops / peak, "traffic": traffic,
                "kernel": "vggt::attn_core_kernel<CoreCfg<2>>", "kernel_ms": core_ms,
                "peak_source": f"{peak_src} bf16_tflops_sustained (back-to-back launches, seconds long)",
                "frac_of_burst_peak": core_tflops / peaks.get("bf16_tflops", peak),
                "prologue_ms": pro_ms,
                "prologue_hbm_gbs": (shape.S * shape.T * shape.H * 64 * 2 * 4) / (pro_ms / 1000) / 1e9}
    # The softmax's exponentials are the kernel's other ceiling: one exp2 per score (N^2 H per call), 7/8 of
    # them on the MUFU unit (16 results/clk/SM), 1/8 as a polynomial on the FMA pipe.
    n_tok = shape.S * shape.T
    exps = float(n_tok) * n_tok * shape.H
    sm_mhz = (clk or {}).get("sm_mhz") or 0.0
    n_sm = torch.cuda.get_device_properties(device).multi_processor_count
    if sm_mhz > 0:
        mufu_peak = 16.0 * n_sm * sm_mhz * 1e6
        roofline["exp"] = {"achieved_per_s": exps / (core_ms / 1000.0), "mufu_share": 7 / 8,
                           "mufu_peak_per_s": mufu_peak,
                           "mufu_frac": exps * 7 / 8 / (core_ms / 1000.0) / mufu_peak,
                           "clock_mhz": sm_mhz}

    # ---- e2e: scenes from pinned host buffers through vggt_attn_host_pipeline: every step's H2D of its
    # qkv and D2H of its output are inside the timed region, on copy streams that overlap the
    # neighbouring steps' kernels (gamma/beta stay resident on the device, as model weights do)
    e2e_iters = max(3, args.steps)
    h_qkv = [torch.empty(qkv.shape, dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
    for h in h_qkv:
        h.copy_(qkv)
    h_out = [torch.empty(out.shape, dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
    pws_bytes = V.vggt_attn_host_pipeline_workspace_size(shape, "global")
    pws = torch.empty(pws_bytes, dtype=torch.uint8, device=device)
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)

    def e2e_run(n):
        V.vggt_attn_host_pipeline("global", shape, [h_qkv[i % 2] for i in range(n)], prm["q_gamma"],
                                  prm["q_beta"], prm["k_gamma"], prm["k_beta"], [h_out[i % 2] for i in range(n)],
                                  pws, pws_bytes, stream, s_in, s_out)

    e2e_run(2)
    torch.cuda.synchronize(device)
    barrier(device)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    e2e_run(e2e_iters)
    t1.record(s_out)
    t1.synchronize()
    assert V.vggt_attn_read_status(pws, stream) == 0
    e2e_ms = reduce_max(t0.elapsed_time(t1) / e2e_iters, device)
    # the same steps one after another on one stream (no overlap), for comparison
    serial_ms = reduce_max(cuda_time_ms(lambda: V.vggt_attn_host_pipeline(
        "global", shape, [h_qkv[0]], prm["q_gamma"], prm["q_beta"], prm["k_gamma"], prm["k_beta"], [h_out[0]],
        pws, pws_bytes, stream, stream, stream), stream, 3), device)
    h2d = qkv.numel() * 2
    d2h = out.numel() * 2
    e2e = {"value": flops * world / (e2e_ms / 1000.0) / 1e12, "unit": UNIT, "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": e2e_iters,
           "api": "vggt_attn_host_pipeline (pinned host in/out, copies on two copy streams)",
           "serial_ms_per_step": serial_ms}
    del h_qkv, h_out, pws

    roofline["frac_clock_normalised"] = clock_normalised_frac(core_tflops, sm_mhz, peaks)
    roofline["clock_note"] = ("frac_clock_normalised = (achieved / this run's median SM MHz) / (sustained peak / "
                              "the SM MHz sampled under load while that peak was measured)")

    # ---- every benchmark configuration: ms/call, the core's TFLOP/s and roofline fraction
    per_config = []
    if not args.no_modes:
        headline = {"call_ms": ms / args.steps, "core_ms": core_ms, "prologue_ms": pro_ms, "sm_mhz": sm_mhz}
        per_config, cfg_clk = config_timings(V, device, stream, peaks, headline)
        roofline["per_config"] = per_config
        roofline["per_config_clocks"] = {k: cfg_clk.get(k) for k in ("sm_mhz", "reasons", "power_w_max")}
    side = {}
    if not args.no_blocks:
        side["blocks"] = block_timings(V, device, stream)
        side["blocks"]["transformer"] = transformer_timings(V, device, stream)
    if not args.no_modes:
        side["sga"] = sga_timings(V, device, stream, qkv, prm, out, ms / args.steps)
        side["sharded_global"] = sharded_timings(V, device, stream, qkv, prm, ms / args.steps)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.cpu_queries)
        if per_config:
            cpu["per_config"] = oracle_config_timings(cpu)

    if world > 1:
        dist.barrier(device_ids=[device.index])
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": headline_config(w, world),
            "pct_of_peak": 100.0 * value / world / peak,
            "e2e": e2e, "roofline": roofline, "gpu_launches": launches, "clocks": clk, "cpu_baseline": cpu}
    if side:   # side measurements (blocks, subsampled and sharded forms) on a line of their own, before the result
        print(json.dumps({"side_measurements": side}), flush=True)
    print(json.dumps(line), flush=True)
    return 0


def run_sharded(args):
    """--sharded: one scene (the 100-frame global workload) split across the ranks by frames; every step is
    query-sharded global attention (vit_attention_b200.sharded.global_attention_sharded: the rank's prologue,
    one NCCL all-gather each of the normalised keys and of the values, then the rank's core over all keys; with
    --overlap the gather runs on a side stream beside the core over the rank's own keys, then the core over the
    other ranks' keys merges with that).
    `value` = the scene's algorithmic flops per step / the max-over-ranks time ("scaling": "strong"); `e2e`
    adds, every step, the H2D of the rank's qkv frames from pinned host memory and the D2H of its output
    rows (serialised with the step on the rank's stream)."""
    import datetime
    import torch
    import torch.distributed as dist
    import vit_attention_b200 as V
    from vit_attention_b200.sharded import global_attention_sharded, overlapped

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    device = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    w = W.workload(HEADLINE)
    frames = scene_frames(w.shape.S, world, rank)
    shape = dataclasses.replace(w.shape, S=len(frames))
    x = W.make_qkv(w.shape, w.seed, w.lowrank, frames)
    prm = W.make_norm_params(w.shape.H, w.seed)
    qkv = torch.from_numpy(x.view(np.int16)).to(device).view(torch.bfloat16)
    g = {k: torch.from_numpy(np.ascontiguousarray(prm[k])).to(device) for k in ("q_gamma", "q_beta", "k_gamma", "k_beta")}
    out = torch.empty((shape.S, shape.T, shape.H, 64), dtype=torch.bfloat16, device=device)
    ws = torch.empty(V.vggt_attn_shard_workspace_size(shape, world), dtype=torch.uint8, device=device)

    def step():
        global_attention_sharded(shape, qkv, g["q_gamma"], g["q_beta"], g["k_gamma"], g["k_beta"], out, ws,
                                 stream=stream, overlap=args.overlap)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    assert V.vggt_attn_read_status(ws, stream) == 0
    clocks = ClockSampler(device.index)
    clocks.start()
    time.sleep(0.4)
    barrier(device)
    torch.cuda.synchronize(device)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    clk = clocks.stop()
    ms = reduce_max(t0.elapsed_time(t1), device)
    assert V.vggt_attn_read_status(ws, stream) == 0
    flops = attention_flops("global", w.shape)                 # the whole scene's work per step
    value = flops * args.steps / (ms / 1000.0) / 1e12
    # e2e: the rank's frames in from pinned host memory and its output rows back, every step
    h_qkv = torch.empty(qkv.shape, dtype=torch.bfloat16, pin_memory=True)
    h_qkv.copy_(qkv)
    h_out = torch.empty(out.shape, dtype=torch.bfloat16, pin_memory=True)
    barrier(device)
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        qkv.copy_(h_qkv, non_blocking=True)
        step()
        h_out.copy_(out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    e2e_ms = reduce_max(e0.elapsed_time(e1), device)
    # the scene's per-rank core alone (the all-gather and the prologue excluded), for the roofline; overlapped,
    # the own keys' launch and the other ranks' launch with the merge
    k_send, v_send, k_all, v_all = V.vggt_attn_shard_buffers(shape, world, ws)
    split = overlapped(world, args.overlap)
    if split:
        def core():
            V.vggt_attn_global_shard_core_local(shape, world, ws, None, stream)
            V.vggt_attn_global_shard_core_remote(shape, world, rank, out, ws, None, stream)
    else:
        def core():
            V.vggt_attn_global_shard_core(shape, world, out, ws, None, stream)
    core_ms = reduce_max(cuda_time_ms(core, stream, max(3, args.steps)), device)
    peaks, peak_src = load_peaks()
    peak = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
    core_tflops = flops / world / (core_ms / 1000.0) / 1e12
    gather_bytes = 2 * (world - 1) * k_send.numel() * 2
    if world > 1:
        dist.barrier(device_ids=[device.index])
        dist.destroy_process_group()
    if rank != 0:
        return 0
    cfg = headline_config(w, world)
    cfg["parallelism"] = (f"query-sharded x{world} over frames, NCCL all-gather of k and v "
                          f"{'beside the own keys attention' if split else 'then the core'} (strong)")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg,
            "e2e": {"value": flops * args.steps / (e2e_ms / 1000.0) / 1e12, "unit": UNIT,
                    "h2d_bytes_per_step": qkv.numel() * 2, "d2h_bytes_per_step": out.numel() * 2,
                    "ms_per_step": e2e_ms / args.steps, "per_rank_bytes": True},
            "roofline": {"bound": "tensor", "achieved": core_tflops, "peak": peak, "unit": "TFLOP/s",
                         "frac": core_tflops / peak, "traffic": None,
                         "kernel": ("vggt::attn_core_kernel<CoreCfg<2, false, true, false, 1>> + "
                                    "attn_core_ranks_kernel<CoreCfg<2, false, true, true, 2>> (one rank's queries: "
                                    "own keys, then the other ranks' keys with the merge)" if split else
                                    "vggt::attn_core_kernel<CoreCfg<2, false, true>> (one rank's queries, all keys)"),
                         "kernel_ms": core_ms, "peak_source": f"{peak_src} bf16_tflops_sustained",
                         "allgather_bytes_per_rank": gather_bytes},
            "gpu_launches": (3 if split else 2) * args.steps, "clocks": clk, "cpu_baseline": None}
    print(json.dumps(line), flush=True)
    return 0


def linear_only(spec: str) -> int:
    """vggt_linear on device-drawn bf16 operands, 3 warm-up + 3 calls, ms per call printed."""
    import torch
    import vit_attention_b200 as V
    M, N, K = (int(v) for v in spec.split(","))
    g = torch.Generator(device="cuda")
    g.manual_seed(99)
    x = torch.randn((M, K), generator=g, device="cuda").to(torch.bfloat16)
    w = (torch.randn((N, K), generator=g, device="cuda") / K ** 0.5).to(torch.bfloat16)
    b = 0.1 * torch.randn(N, generator=g, device="cuda")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    fn = lambda: V.vggt_linear(x, w, b, y, ws)
    for _ in range(3):
        fn()
    ms = cuda_time_ms(fn, torch.cuda.current_stream(), 3)
    assert V.vggt_attn_read_status(ws) == 0
    print(json.dumps({"linear": [M, N, K], "ms": ms, "tflops": 2.0 * M * N * K / (ms / 1000) / 1e12}), flush=True)
    return 0


def sga_timings(V, device, stream, qkv, prm, out, global_ms):
    """Subsampled global attention on the headline workload (kept-key grid s x s):
    ms per call, speedup over the exact global call, TFLOP/s over the kept keys."""
    import torch
    w = W.workload(HEADLINE)
    shape = w.shape
    res = {}
    n = shape.S * shape.T
    for s_ in (2, 3):
        ws = torch.empty(V.vggt_attn_sga_workspace_size(shape, s_, s_), dtype=torch.uint8, device=device)
        fn = lambda: V.vggt_attn_global_sga(shape, s_, s_, qkv, prm["q_gamma"], prm["q_beta"], prm["k_gamma"],
                                            prm["k_beta"], out, ws, None, stream)
        for _ in range(2):
            fn()
        t = cuda_time_ms(fn, stream, 5)
        assert V.vggt_attn_read_status(ws, stream) == 0
        nk = shape.S * (shape.n_special + ((shape.grid_h + s_ - 1) // s_) * ((shape.grid_w + s_ - 1) // s_))
        res[f"grid_{s_}x{s_}"] = {"ms": t, "kept_keys": nk, "speedup_vs_global": global_ms / t,
                                 "tflops_over_kept_keys": 4.0 * n * nk * 64 * shape.H / (t / 1000) / 1e12}
        # descriptor attention over the same number of keys (window means instead of window corners)
        fd = lambda: V.vggt_attn_global_desc(shape, s_, s_, qkv, prm["q_gamma"], prm["q_beta"], prm["k_gamma"],  # noqa: E731
                                             prm["k_beta"], out, ws, None, stream)
        fd()
        td = cuda_time_ms(fd, stream, 5)
        assert V.vggt_attn_read_status(ws, stream) == 0
        res[f"desc_{s_}x{s_}"] = {"ms": td, "descriptors": nk, "speedup_vs_global": global_ms / td,
                                 "tflops_over_descriptors": 4.0 * n * nk * 64 * shape.H / (td / 1000) / 1e12}
        del ws
    return res


def sharded_timings(V, device, stream, qkv, prm, global_ms):
    """Query-sharded global attention on the headline workload, one rank's work for world sizes 1-8 on this
    GPU: the rank's prologue over its S/world frames and its core over all keys (the all-gather between
    them is not timed: one GPU here); the keys come from the whole scene's gathered buffer, filled once."""
    import torch
    w = W.workload(HEADLINE)
    res = {}
    for world in (1, 2, 4, 5):                     # divisors of the 100 frames
        local = dataclasses.replace(w.shape, S=w.shape.S // world)
        ws = torch.empty(V.vggt_attn_shard_workspace_size(local, world), dtype=torch.uint8, device=device)
        qkv_r = qkv[:local.S]
        out_r = torch.empty((local.S, local.T, local.H, 64), dtype=torch.bfloat16, device=device)
        pro = lambda: V.vggt_attn_global_shard_prologue(local, world, qkv_r, prm["q_gamma"], prm["q_beta"],  # noqa: E731
                                                       prm["k_gamma"], prm["k_beta"], ws, None, stream)
        core = lambda: V.vggt_attn_global_shard_core(local, world, out_r, ws, None, stream)  # noqa: E731
        pro()
        k_send, v_send, k_all, v_all = V.vggt_attn_shard_buffers(local, world, ws)
        for r in range(world):                     # stand-in for the all-gather: the rank's block, repeated
            k_all[r * k_send.shape[0]:(r + 1) * k_send.shape[0]].copy_(k_send)
            v_all[r * v_send.shape[0]:(r + 1) * v_send.shape[0]].copy_(v_send)
        core()
        t_pro = cuda_time_ms(pro, stream, 3)
        t_core = cuda_time_ms(core, stream, 3)
        assert V.vggt_attn_read_status(ws, stream) == 0
        # fused form: the same keys read in place from `world` per-rank buffers (here all on this GPU)
        ks = [k_send] * world
        vs = [v_send] * world
        fused = lambda: V.vggt_attn_global_shard_core_peers(local, world, ks, vs, out_r, ws, None, stream)  # noqa: E731
        fused()
        t_fused = cuda_time_ms(fused, stream, 3)
        assert V.vggt_attn_read_status(ws, stream) == 0
        gather_bytes = 2 * (world - 1) * k_send.numel() * 2          # k and v blocks received per rank
        res[f"world_{world}"] = {"rank_prologue_ms": t_pro, "rank_core_ms": t_core, "rank_core_fused_ms": t_fused,
                                 "rank_compute_ms": t_pro + t_core,
                                 "speedup_vs_1gpu_global": global_ms / (t_pro + t_core),
                                 "allgather_bytes_per_rank": gather_bytes,
                                 "allgather_ms_at_770GBs": gather_bytes / 770e9 * 1e3}
        if world >= 2:
            # overlapped form: the own keys' core (beside the all-gather), then the other ranks' keys with the merge
            local_core = lambda: V.vggt_attn_global_shard_core_local(local, world, ws, None, stream)  # noqa: E731
            remote_core = lambda: V.vggt_attn_global_shard_core_remote(local, world, 0, out_r, ws, None, stream)  # noqa: E731
            local_core()
            remote_core()
            t_local = cuda_time_ms(local_core, stream, 3)
            t_remote = cuda_time_ms(remote_core, stream, 3)
            assert V.vggt_attn_read_status(ws, stream) == 0
            gather_ms = gather_bytes / 770e9 * 1e3
            res[f"world_{world}"].update({"rank_core_local_ms": t_local, "rank_core_remote_ms": t_remote,
                                          "rank_core_split_ms": t_local + t_remote,
                                          "allgather_exposed_ms_at_770GBs": max(0.0, gather_ms - t_local)})
        del ws, out_r
    return res


def block_timings(V, device, stream):
    """One attention block (QKV GEMM, QK-norm/RoPE prologue, attention core,
    output projection; vggt_attn_block) on token features, for the S=100 global
    and the S=500 frame workloads: ms per block and per stage, the GEMMs'
    TFLOP/s, and the fused QKV projection (GEMM with the prologue in its
    epilogue) for comparison (device-drawn inputs, random weights of the model's
    shapes)."""
    import torch
    res = {}
    g = torch.Generator(device=device)
    g.manual_seed(4321)
    for label, idx, mode in (("global_S100", 3, "global"), ("frame_S500", 4, "frame"), ("register_S500", 4, "register")):
        shape = W.workload(idx).shape
        M, C = shape.S * shape.T, shape.H * 64
        x = torch.randn((M, C), generator=g, device=device).to(torch.bfloat16)
        w_qkv = (torch.randn((3 * C, C), generator=g, device=device) / C ** 0.5).to(torch.bfloat16)
        w_out = (torch.randn((C, C), generator=g, device=device) / C ** 0.5).to(torch.bfloat16)
        b_qkv = 0.1 * torch.randn(3 * C, generator=g, device=device)
        b_out = 0.1 * torch.randn(C, generator=g, device=device)
        prm = {k: (1.0 if "gamma" in k else 0.0) + 0.1 * torch.randn((shape.H, 64), generator=g, device=device)
               for k in ("q_gamma", "q_beta", "k_gamma", "k_beta")}
        qkv = torch.empty((shape.S, shape.T, 3, shape.H, 64), dtype=torch.bfloat16, device=device)
        attn = torch.empty((M, C), dtype=torch.bfloat16, device=device)
        y = torch.empty((M, C), dtype=torch.bfloat16, device=device)
        ws = torch.empty(V.vggt_attn_workspace_size(shape, mode), dtype=torch.uint8, device=device)
        gq, bq, gk, bk = prm["q_gamma"], prm["q_beta"], prm["k_gamma"], prm["k_beta"]
        stages = {
            "block": lambda: V.vggt_attn_block(mode, shape, x, w_qkv, b_qkv, gq, bq, gk, bk, w_out, b_out, qkv, attn,
                                               y, ws, None, stream),
            "qkv_gemm": lambda: V.vggt_linear(x, w_qkv, b_qkv, qkv.view(M, 3 * C), ws, None, stream),
            "prologue": lambda: V.vggt_attn_prologue(mode, shape, qkv, gq, bq, gk, bk, ws, None, stream),
            "core": lambda: V.vggt_attn_core(mode, shape, qkv, attn, ws, None, stream),
            "out_proj": lambda: V.vggt_linear(attn, w_out, b_out, y, ws, None, stream),
            "qkv_proj_fused": lambda: V.vggt_attn_qkv_proj(mode, shape, x, w_qkv, b_qkv, gq, bq, gk, bk, qkv, ws,
                                                           None, stream),
        }
        if mode == "register":   # the block runs on the gathered special tokens; time it whole
            stages = {"block": stages["block"]}
        entry = {}
        for name, fn in stages.items():
            for _ in range(2):
                fn()
            entry[name + "_ms"] = cuda_time_ms(fn, stream, 5 if mode == "global" else 10)
        assert V.vggt_attn_read_status(ws, stream) == 0
        res[label] = entry
        if mode == "register":
            del x, qkv, attn, y, ws
            continue
        entry["qkv_gemm_tflops"] = 2.0 * M * 3 * C * C / (entry["qkv_gemm_ms"] / 1000) / 1e12
        entry["out_proj_tflops"] = 2.0 * M * C * C / (entry["out_proj_ms"] / 1000) / 1e12
        entry["qkv_proj_fused_tflops"] = 2.0 * M * 3 * C * C / (entry["qkv_proj_fused_ms"] / 1000) / 1e12
        del x, qkv, attn, y, ws
    res["layer_S500_register_plus_frame_block_ms"] = res["register_S500"]["block_ms"] + res["frame_S500"]["block_ms"]
    return res


def random_block_weights(H: int, g, device):
    """Device-drawn weights of one transformer block (the oracle's recipe: N(0, 1/fan_in) bf16 matrices,
    gammas and LayerScales 1 + 0.1 N(0, 1), betas and biases 0.1 N(0, 1))."""
    import torch
    C = H * 64

    def mat(n_out, n_in):
        return (torch.randn((n_out, n_in), generator=g, device=device) / n_in ** 0.5).to(torch.bfloat16)

    def vec(n, centre):
        return centre + 0.1 * torch.randn(n, generator=g, device=device)

    return dict(norm1_gamma=vec(C, 1.0), norm1_beta=vec(C, 0.0), w_qkv=mat(3 * C, C), b_qkv=vec(3 * C, 0.0),
                q_gamma=vec(C, 1.0), q_beta=vec(C, 0.0), k_gamma=vec(C, 1.0), k_beta=vec(C, 0.0),
                w_proj=mat(C, C), b_proj=vec(C, 0.0), ls1=vec(C, 1.0), norm2_gamma=vec(C, 1.0),
                norm2_beta=vec(C, 0.0), w_fc1=mat(4 * C, C), b_fc1=vec(4 * C, 0.0), w_fc2=mat(C, 4 * C),
                b_fc2=vec(C, 0.0), ls2=vec(C, 1.0))


def transformer_timings(V, device, stream):
    """Whole transformer blocks (LayerNorm, QKV GEMM, attention, projection + LayerScale residual,
    LayerNorm, fc1 + GELU, fc2 + LayerScale residual; vggt_block_forward) per mode at S=100 and S=500,
    the two kinds of layer (frame + global, frame + register), and the 24-layer alternating schedule
    (register blocks at layers 2, 6, 9, 14, 20; vggt_aggregator_forward) at S=100 (device-drawn inputs,
    random weights of the model's shapes)."""
    import torch
    res = {}
    g = torch.Generator(device=device)
    g.manual_seed(8765)
    eps = 1e-6
    for idx in (3, 4):
        shape = W.workload(idx).shape
        M, C = shape.S * shape.T, shape.H * 64
        x = torch.randn((M, C), generator=g, device=device).to(torch.bfloat16)
        ws = torch.empty(V.vggt_aggregator_workspace_size(shape), dtype=torch.uint8, device=device)
        w = random_block_weights(shape.H, g, device)
        entry = {}
        for mode in ("frame", "global", "register"):
            if idx == 4 and mode == "global":
                continue                        # S=500 runs register layers only
            fn = lambda m=mode: V.vggt_block_forward(m, shape, x, w, eps, ws, None, stream)  # noqa: E731
            fn()
            entry[f"{mode}_block_ms"] = cuda_time_ms(fn, stream, 3 if mode == "global" else 5)
        assert V.vggt_attn_read_status(ws, stream) == 0
        if idx == 3:
            entry["global_layer_ms"] = entry["frame_block_ms"] + entry["global_block_ms"]
            n = 24
            fws = [random_block_weights(shape.H, g, device) for _ in range(n)]
            iws = [random_block_weights(shape.H, g, device) for _ in range(n)]
            regs = [2, 6, 9, 14, 20]
            agg = lambda: V.vggt_aggregator_forward(shape, x, fws, iws, regs, eps, ws, None, stream)  # noqa: E731
            agg()
            entry["aggregator_24_layers_ms"] = cuda_time_ms(agg, stream, 1)
            assert V.vggt_attn_read_status(ws, stream) == 0
            del fws, iws
        entry["register_layer_ms"] = entry["frame_block_ms"] + entry["register_block_ms"]
        del x, ws, w
        # Camera-head trunk: 4 blocks over the S x 17 special tokens of the last layer's
        # 2 x 1024-wide features (32 heads of 64).
        fshape = dataclasses.replace(shape, H=2 * shape.H)
        feats = torch.randn((M, 2 * C), generator=g, device=device).to(torch.bfloat16)
        tok = torch.empty((shape.S * shape.n_special, 2 * C), dtype=torch.bfloat16, device=device)
        ws = torch.empty(V.vggt_camera_trunk_workspace_size(fshape), dtype=torch.uint8, device=device)
        cws = [random_block_weights(fshape.H, g, device) for _ in range(4)]
        cam = lambda: V.vggt_camera_trunk_forward(fshape, feats, tok, cws, eps, ws, None, stream)  # noqa: E731
        cam()
        entry["camera_trunk_4_blocks_ms"] = cuda_time_ms(cam, stream, 5)
        assert V.vggt_attn_read_status(ws, stream) == 0
        res[f"S{shape.S}"] = entry
        del feats, tok, ws, cws
    return res


# The benchmark's configurations: (label, workload index, mode).  Workload 3 is the headline, timed above.
CONFIG_RUNS = [("cfg0_global_S2_T69_H4", 0, "global"), ("cfg1_frame_S24", 1, "frame"),
               ("cfg2_global_S24_N24744", 2, "global"), ("cfg3_global_S100_N103100", 3, "global"),
               ("cfg4a_register_S500", 4, "register"), ("cfg4b_frame_S500", 4, "frame")]


def clock_normalised_frac(tflops, run_mhz, peaks):
    """Achieved TFLOP/s per MHz of the run's median SM clock, over the sustained GEMM peak per MHz of the
    clock sampled under load while that peak was measured (None without both clocks)."""
    peak_mhz = ((peaks.get("clocks_under_load") or {}).get("sm_mhz_median"))
    peak = peaks.get("bf16_tflops_sustained")
    if not run_mhz or not peak_mhz or not peak:
        return None
    return (tflops / run_mhz) / (peak / peak_mhz)


def config_timings(V, device, stream, peaks, headline):
    """ms per call (QK-norm/RoPE prologue + attention core), the core and the prologue alone, and the
    core's roofline fraction, for every benchmark configuration; the S=500 layer (register + frame call).
    Inputs are drawn on the device with the workload's shape and value distribution (timing only; the
    seeded host inputs are the parity tests' business).  Configs whose inputs fit in L2 (the tiny one)
    are timed back to back, as a latency figure."""
    import torch
    peak = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
    burst = peaks.get("bf16_tflops", peak)
    g = torch.Generator(device=device)
    g.manual_seed(1234)
    clocks = ClockSampler(device.index)
    clocks.start()
    rows, cache = [], {}
    for label, idx, mode in CONFIG_RUNS:
        w = W.workload(idx)
        shape = w.shape
        if idx == 3:
            call_ms, core_ms, pro_ms = headline["call_ms"], headline["core_ms"], headline["prologue_ms"]
        else:
            if idx not in cache:
                cache.clear()
                qkv = torch.randn((shape.S, shape.T, 3, shape.H, 64), generator=g, device=device,
                                  dtype=torch.float32).to(torch.bfloat16)
                prm = [(1.0 if k % 2 == 0 else 0.0) + 0.1 * torch.randn((shape.H, 64), generator=g, device=device)
                       for k in range(4)]
                cache[idx] = (qkv, prm, torch.empty((shape.S, shape.T, shape.H, 64), dtype=torch.bfloat16,
                                                    device=device))
            qkv, prm, out = cache[idx]
            wsb = V.vggt_attn_workspace_size(shape, mode)
            ws = torch.empty(wsb, dtype=torch.uint8, device=device)
            call = lambda: V.attend(mode, shape, qkv, *prm, out, ws, stream)  # noqa: E731
            for _ in range(3):
                call()
            iters = 200 if idx == 0 else 20
            call_ms = cuda_time_ms(call, stream, iters)
            core_ms = cuda_time_ms(lambda: V.vggt_attn_core(mode, shape, qkv, out, ws, wsb, stream), stream, iters)
            pro_ms = cuda_time_ms(lambda: V.vggt_attn_prologue(mode, shape, qkv, *prm, ws, wsb, stream), stream,
                                  iters)
            assert V.vggt_attn_read_status(ws, stream) == 0
            del ws
        f = attention_flops(mode, shape)
        core_tf = f / (core_ms / 1000) / 1e12
        row = {"config": label, "mode": mode, "ms": call_ms, "core_ms": core_ms, "prologue_ms": pro_ms,
               "tflops": f / (call_ms / 1000) / 1e12, "core_tflops": core_tf, "frac": core_tf / peak,
               "frac_burst": core_tf / burst,
               "prologue_hbm_gbs": io_bytes(mode, shape) / (pro_ms / 1000) / 1e9}
        if mode == "register":
            row["gbs_min_io"] = io_bytes(mode, shape) / (call_ms / 1000) / 1e9
        rows.append(row)
    cache.clear()
    clk = clocks.stop()
    mhz = clk.get("sm_mhz")
    for row in rows:
        run_mhz = headline["sm_mhz"] if row["config"].startswith("cfg3") else mhz
        row["frac_clock_normalised"] = clock_normalised_frac(row["core_tflops"], run_mhz, peaks)
        row["sm_mhz"] = run_mhz
    by = {r["config"]: r for r in rows}
    layer = by["cfg4a_register_S500"]["ms"] + by["cfg4b_frame_S500"]["ms"]
    rows.append({"config": "cfg4_layer_S500_register_plus_frame", "mode": "layer", "ms": layer,
                 "tflops": (attention_flops("register", W.workload(4).shape) +
                            attention_flops("frame", W.workload(4).shape)) / (layer / 1000) / 1e12})
    return rows, clk


def oracle_config_timings(headline_cpu):
    """The fp64 oracle timed on this host for every configuration: in full where that takes seconds, else on a
    seeded sample with the full time extrapolated by the ratio of algorithmic work (labelled)."""
    import oracle as O
    from threadpoolctl import threadpool_info
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    res = []

    def timed(fn):
        t0 = time.perf_counter()
        fn()
        return time.perf_counter() - t0

    def entry(label, mode, shape, sample, seconds, frac_of_work):
        full = seconds / frac_of_work
        return {"config": label, "mode": mode, "sample": sample, "seconds": seconds, "full_seconds": full,
                "extrapolated": frac_of_work < 1.0, "tflops": attention_flops(mode, shape) / full / 1e12,
                "cores": threads}

    for label, idx, mode in CONFIG_RUNS:
        w = W.workload(idx)
        shape = w.shape
        if idx == 3:
            res.append(entry(label, mode, shape, headline_cpu["sample"], headline_cpu["seconds"],
                             headline_cpu["queries"] / (shape.S * shape.T)))
            continue
        x = _ORACLE_INPUTS.get(w.name)
        if x is None:
            x = _ORACLE_INPUTS.setdefault(w.name, W.make_inputs(w))
        if mode == "global" and idx == 2:
            q = W.query_subset(shape.S * shape.T, 1024, w.seed)
            dt = timed(lambda: O.attn_global(shape, x, q))
            res.append(entry(label, mode, shape, "1024 seeded queries x 16 heads over all 24,744 keys", dt,
                             1024 / (shape.S * shape.T)))
        elif mode == "frame" and idx == 4:
            frames = np.sort(np.random.default_rng([w.seed, 5]).choice(shape.S, 4, replace=False))
            q = (frames[:, None] * shape.T + np.arange(shape.T)[None, :]).reshape(-1)
            dt = timed(lambda: O.attn_frame(shape, x, q))
            res.append(entry(label, mode, shape, "every query of 4 seeded frames (of 500)", dt, 4 / shape.S))
        else:
            dt = timed(lambda: O.attn_mode(mode, shape, x))
            res.append(entry(label, mode, shape, "full", dt, 1.0))
    _ORACLE_INPUTS.clear()
    return res


def run_one(args) -> int:
    """One attention mode (or one transformer block, or subsampled / descriptor global attention) on
    device-drawn inputs of a workload's shape: one warm-up call, then --calls timed calls; prints ms per call.
    A small driver for profiling a single kernel under ncu (no side measurements, no oracle)."""
    import torch
    import vit_attention_b200 as V
    mode = args.one
    torch.cuda.set_device(0)
    shape = W.workload(args.workload).shape
    if args.frames > 0:
        shape = dataclasses.replace(shape, S=args.frames)
    if args.patch_grid is not None:   # e.g. 0 0: frames of special tokens only (register mode's whole input)
        gh, gw = args.patch_grid
        shape = dataclasses.replace(shape, grid_h=gh, grid_w=gw, T=shape.n_special + gh * gw)
    g = torch.Generator(device="cuda")
    g.manual_seed(1234)
    H, C = shape.H, shape.H * 64
    if args.block:
        w = random_block_weights(H, g, torch.device("cuda"))
        x = torch.randn((shape.S * shape.T, C), generator=g, device="cuda").to(torch.bfloat16)
        ws = torch.empty(V.vggt_block_workspace_size(shape, mode), dtype=torch.uint8, device="cuda")

        def call():
            V.vggt_block_forward(mode, shape, x, w, 1e-6, ws)
    else:
        qkv = torch.randn((shape.S, shape.T, 3, H, 64), generator=g, device="cuda").to(torch.bfloat16)
        prm = [(1.0 if k % 2 == 0 else 0.0) + 0.1 * torch.randn((H, 64), generator=g, device="cuda")
               for k in range(4)]
        out = torch.empty((shape.S, shape.T, H, 64), dtype=torch.bfloat16, device="cuda")
        if args.sga or args.desc:
            sz = args.sga or args.desc
            fn = V.vggt_attn_global_sga if args.sga else V.vggt_attn_global_desc
            ws = torch.empty(V.vggt_attn_sga_workspace_size(shape, sz, sz), dtype=torch.uint8, device="cuda")

            def call():
                fn(shape, sz, sz, qkv, *prm, out, ws)
        else:
            ws = torch.empty(V.vggt_attn_workspace_size(shape, mode), dtype=torch.uint8, device="cuda")

            def call():
                V.attend(mode, shape, qkv, *prm, out, ws)
    call()
    torch.cuda.synchronize()
    ms = cuda_time_ms(call, torch.cuda.current_stream(), max(args.calls, 1))
    status = V.vggt_attn_read_status(ws)
    print(json.dumps({"one": mode, "block": args.block, "sga": args.sga, "desc": args.desc, "S": shape.S,
                      "T": shape.T, "H": H, "ms_per_call": ms, "status": status}), flush=True)
    return 0 if status == 0 else 1


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-queries", type=int, default=512, help="oracle sample size of the CPU baseline")
    ap.add_argument("--ref-queries", type=int, default=16, help="oracle queries per step of --impl reference")
    ap.add_argument("--workload", type=int, default=HEADLINE,
                    help="index of a global-mode workload (default: the S=100 headline; 2 = S=24 for profiling)")
    ap.add_argument("--no-modes", action="store_true")
    ap.add_argument("--no-blocks", action="store_true", help="skip the attention-block (projections + core) timings")
    ap.add_argument("--linear-only", default=None, metavar="M,N,K",
                    help="run vggt_linear on an M x N x K problem a few times and exit (a small case for ncu)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sharded", action="store_true",
                    help="one 100-frame scene split across the ranks by frames: query-sharded global attention with "
                         "an NCCL all-gather of the keys and values (strong scaling; the ranks must divide 100)")
    ap.add_argument("--overlap", action="store_true",
                    help="with --sharded: the all-gather on a side stream beside the core over the rank's own keys, "
                         "then the other ranks' keys with a merge (2 to 9 ranks)")
    ap.add_argument("--one", choices=("frame", "global", "register"), default=None,
                    help="run only this mode on --workload's shape (--frames, --calls, --block, --sga, --desc) and "
                         "exit: a small case for ncu")
    ap.add_argument("--frames", type=int, default=0, help="with --one: override the frame count S")
    ap.add_argument("--calls", type=int, default=3, help="with --one: timed calls after one warm-up call")
    ap.add_argument("--patch-grid", type=int, nargs=2, default=None, metavar=("H", "W"),
                    help="with --one: override the patch grid (0 0: special tokens only, a small input that gives "
                         "register mode its full problem)")
    ap.add_argument("--block", action="store_true", help="with --one: a whole transformer block")
    ap.add_argument("--sga", type=int, default=0, help="with --one global: subsampled global attention, s x s grid")
    ap.add_argument("--desc", type=int, default=0, help="with --one global: descriptor attention, s x s windows")
    args = ap.parse_args()
    if args.linear_only:
        return linear_only(args.linear_only)
    if args.one:
        return run_one(args)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.sharded:
        return run_sharded(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
