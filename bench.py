#!/usr/bin/env python
"""Benchmark of the tiled attention forward pass on B200.

One step = one pass of the whole hot path over the headline workload
(B=4, H=32, N=4096, d=128, causal, bf16; scale 1/sqrt(128)) in int8_qk mode:
K-mean / smoothing / INT8 quantisation pre-pass, then the fused INT8-QK^T /
16-bit-PV attention kernel.  bf16_exact is timed the same way and reported
under "modes".  Metric: attention FLOPs 4*B*H*N^2*d/2 per step over device
time (TFLOP/s), whole job (sum over ranks / max time over ranks).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                  [--config 2] [--no-e2e] [--no-cpu-baseline]

Multi-GPU: one process per GPU (torchrun); each rank runs its own independent
batch of the workload (the (batch, head) units share nothing), so no
collective is on the data path and scaling is weak.  ``--impl reference``
times the CPU float64 oracle (the only reference this method has) on a
bounded sample of the same workload.
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from attn_workloads import (APB_WORKLOADS, DECODE_WORKLOADS, WORKLOADS, decode_bytes, make_apb_inputs,  # noqa: E402
                            make_decode_inputs, make_inputs)


KERNEL_SOURCES = ("tiled_attention_22_b200/csrc/attn_fwd_kernels.cuh", "tiled_attention_22_b200/csrc/ptx.cuh",
                  "tiled_attention_22_b200/csrc/attn_fwd_launch.cuh", "tiled_attention_22_b200/csrc/tma_host.cuh",
                  "tiled_attention_22_b200/csrc/attn_fwd_persistent.cuh")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_fwd_kernel_traffic_mha_causal_b4_h32_n4096_d128.txt")


def _kernel_source_hash():
    import hashlib

    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def _measured_traffic(mode):
    """DRAM bytes per launch of the fused kernel from the committed ncu summary, or None when the
    kernel sources changed since those counters were taken (or no summary exists)."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    fields = {}
    with open(TRAFFIC_FILE) as f:
        for line in f:
            if "=" in line and not line.lstrip().startswith("#"):
                key, val = line.split("=", 1)
                fields[key.strip()] = val.strip()
    if fields.get("kernel_source_sha256") != _kernel_source_hash():
        return None
    val = fields.get(f"{mode}_dram_bytes_per_launch")
    return int(val) if val else None


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16": d["bf16_tflops"], "bf16_sustained": d["bf16_tflops_sustained"],
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi samples taken while the timed region runs (200 ms period)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.rows = []
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), line.strip()))

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        inside = [r for t, r in self.rows if self.t0 is not None and self.t0 <= t <= (self.t1 or t)]
        rows = inside or [r for _, r in self.rows]
        sm, mx, reasons = [], None, set()
        for r in rows:
            parts = [p.strip() for p in r.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "in_timed_region": bool(inside)}


def _dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def _barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def _max_over_ranks(x, world, device="cuda"):
    """Maximum of a per-rank scalar (the job's time is its slowest rank's time)."""
    if world == 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(local_ms, flops_per_rank, world, device="cuda"):
    """Whole-job throughput: the work of all ranks over the slowest rank's time.
    Returns (max_ms, TFLOP/s)."""
    ms = _max_over_ranks(local_ms, world, device)
    return ms, flops_per_rank * world / (ms * 1e-3) / 1e12


def cpu_baseline(w, budget_s=15.0):
    """The CPU oracle (float64 numpy, as it stands) on a bounded sample of the workload: the int8
    emulation pre-pass and the attention of whole heads, as many heads as fit in the budget."""
    import numpy as np

    import oracle

    cores = len(os.sched_getaffinity(0))
    q, k, v = make_inputs(w)
    G = w.Hq // w.Hkv
    t0 = time.perf_counter()
    flops = 0.0
    heads = 0
    for b in range(w.B):
        for h in range(w.Hq):
            g = h // G
            qs, ks, vs = q[b:b + 1, h:h + 1], k[b:b + 1, g:g + 1], v[b:b + 1, g:g + 1]
            q8, sq, k8, sk, mean, bias = oracle.prepass(qs, ks, w.scale)
            oracle.attention_int8(q8, sq, k8, sk, bias, vs, w.scale, w.causal)
            flops += 4.0 * w.N * w.N * w.d / (2.0 if w.causal else 1.0)
            heads += 1
            if time.perf_counter() - t0 > budget_s:
                break
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    del np
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{heads} of {w.B * w.Hq} (batch, head) units, all {w.N} rows each: INT8 emulation "
                      f"pre-pass + float64 attention, {dt:.1f} s", "seconds": dt}


def run_reference(args, w, world, rank):
    line = {"metric": f"attention fwd TFLOP/s (int8_qk step) on {w.name}", "impl": "reference",
            "unit": "TFLOP/s", "higher_is_better": True, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup}
    if rank != 0:
        return None
    import oracle

    q, k, v = make_inputs(w)
    G = w.Hq // w.Hkv
    per_step_heads = 1
    total_flops = 0.0
    t_total = 0.0
    idx = 0
    for step in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        flops = 0.0
        for _ in range(per_step_heads):
            b, h = divmod(idx % (w.B * w.Hq), w.Hq)
            idx += 1
            g = h // G
            qs, ks, vs = q[b:b + 1, h:h + 1], k[b:b + 1, g:g + 1], v[b:b + 1, g:g + 1]
            q8, sq, k8, sk, mean, bias = oracle.prepass(qs, ks, w.scale)
            oracle.attention_int8(q8, sq, k8, sk, bias, vs, w.scale, w.causal)
            flops += 4.0 * w.N * w.N * w.d / (2.0 if w.causal else 1.0)
        dt = time.perf_counter() - t0
        if step >= args.warmup:
            total_flops += flops
            t_total += dt
    value = total_flops / t_total / 1e12
    cores = len(os.sched_getaffinity(0))
    line.update({"value": value, "ms_per_step": 1e3 * t_total / args.steps, "scaling": "weak",
                 "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                 "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d,
                            "causal": w.causal},
                 "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                  "sample": f"each step: {per_step_heads} (batch, head) unit of the workload, "
                                            f"all {w.N} rows, INT8 emulation pre-pass + float64 attention"},
                 "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}})
    return line


def run_native(args, w, world, rank, local):
    import tiled_attention_22_b200 as ta

    dev = torch.device("cuda", local)
    q, k, v = make_inputs(w)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.N, w.d
    o = torch.empty_like(qd)
    lse = torch.empty((B, Hq, N), device=dev, dtype=torch.float32)
    T = (N + 127) // 128
    pre = dict(q8=torch.empty((B, Hq, N, d), device=dev, dtype=torch.int8),
               sq=torch.empty((B, Hq, T), device=dev, dtype=torch.float32),
               k8=torch.empty((B, Hkv, N, d), device=dev, dtype=torch.int8),
               sk=torch.empty((B, Hkv, T), device=dev, dtype=torch.float32),
               kmean=torch.empty((B, Hkv, d), device=dev, dtype=torch.float32),
               lse_bias=torch.empty((B, Hq, N), device=dev, dtype=torch.float32))
    scratch = torch.empty(ta.attn_quant_scratch_bytes(B, Hkv, N, d), device=dev, dtype=torch.uint8)
    pre8 = dict(pre, q8=pre["q8"].view(torch.uint8), k8=pre["k8"].view(torch.uint8))
    stream = torch.cuda.current_stream()
    flops = w.flops()

    def step_int8(ev=None):
        if ev:
            ev[0].record(stream)
        ta.attn_quant_smooth_k(qd, kd, scale=w.scale, scratch=scratch, stream=stream, out=pre)
        if ev:
            ev[1].record(stream)
        ta.attn_fwd_int8_quantized(pre, vd, causal=w.causal, scale=w.scale, out=o, lse=lse, stream=stream)
        if ev:
            ev[2].record(stream)

    def step_fp8(ev=None):
        if ev:
            ev[0].record(stream)
        ta.attn_quant_smooth_k_fp8(qd, kd, scale=w.scale, scratch=scratch, stream=stream, out=pre8)
        if ev:
            ev[1].record(stream)
        ta.attn_fwd_fp8_quantized(pre8, vd, causal=w.causal, scale=w.scale, out=o, lse=lse, stream=stream)
        if ev:
            ev[2].record(stream)

    def step_bf16(ev=None):
        if ev:
            ev[0].record(stream)
        ta.attn_fwd(qd, kd, vd, causal=w.causal, scale=w.scale, mode="bf16_exact", out=o, lse=lse, stream=stream)
        if ev:
            ev[1].record(stream)

    results = {}
    sampler = ClockSampler(int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[0])
                           if os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")[0].isdigit() else local)
    sampler.start()
    time.sleep(0.3)
    for mode, fn, nk in (("int8_qk", step_int8, 2), ("bf16_exact", step_bf16, 1), ("fp8_qk", step_fp8, 2)):
        if mode not in args.modes.split(","):
            continue
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        _barrier(world)
        torch.cuda.synchronize()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)] for _ in range(args.steps)]
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if mode == "int8_qk":
            sampler.mark("t0")
        start.record(stream)
        for s in range(args.steps):
            fn(evs[s])
        end.record(stream)
        torch.cuda.synchronize()
        if mode == "int8_qk":
            sampler.mark("t1")
        _barrier(world)
        torch.cuda.synchronize()
        ms, tflops = whole_job_rate(start.elapsed_time(end), flops * args.steps, world)
        if ta.attn_check_status() != 0:
            raise RuntimeError("device-side wait timed out during the benchmark")
        kern = [statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs) for i in range(nk)]
        results[mode] = {"ms_total": ms, "ms_per_step": ms / args.steps, "tflops": tflops, "kernel_ms": kern}
    clocks = sampler.stop()

    # end to end through the public C ABI with host buffers: H2D q,k,v + forward + D2H o, lse
    e2e = None
    if not args.no_e2e:
        qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
        oh = torch.empty_like(qh).pin_memory()
        lh = torch.empty((B, Hq, N), dtype=torch.float32).pin_memory()
        ws = torch.empty(ta.attn_workspace_bytes(B, Hq, Hkv, N, d, "int8_qk"), device=dev, dtype=torch.uint8)
        e_steps = max(3, min(args.steps, 50))
        for _ in range(2):
            ta.attn_fwd_host(qh, kh, vh, oh, lh, qd, kd, vd, o, lse, causal=w.causal, scale=w.scale,
                             mode="int8_qk", workspace=ws, stream=stream)
        _barrier(world)
        torch.cuda.synchronize()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for _ in range(e_steps):
            ta.attn_fwd_host(qh, kh, vh, oh, lh, qd, kd, vd, o, lse, causal=w.causal, scale=w.scale,
                             mode="int8_qk", workspace=ws, stream=stream)
        s1.record(stream)
        torch.cuda.synchronize()
        ems, e2e_tflops = whole_job_rate(s0.elapsed_time(s1), flops * e_steps, world)
        e2e = {"value": e2e_tflops, "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(3 * q.numel() * q.element_size()),
               "d2h_bytes_per_step": int(o.numel() * o.element_size() + lse.numel() * 4),
               "steps": e_steps, "ms_per_step": ems / e_steps}

    peaks = _peaks()
    nan = {"ms_total": float("nan"), "ms_per_step": float("nan"), "tflops": float("nan"),
           "kernel_ms": [float("nan"), float("nan")]}
    r8 = results.get("int8_qk", nan)
    rb = results.get("bf16_exact", nan)
    rf = results.get("fp8_qk", nan)
    long_region = r8["ms_total"] > 1000.0
    bf16_peak = peaks["bf16_sustained"] if long_region else peaks["bf16"]
    mixed_peak = bf16_peak * 4.0 / 3.0  # QK^T at the INT8 rate (2x bf16, nominal ratio), PV at the bf16 rate
    fused_ms = r8["kernel_ms"][1]
    achieved = flops / (fused_ms * 1e-3) / 1e12
    line = {
        "metric": f"attention fwd TFLOP/s (int8_qk step) on {w.name}",
        "value": r8["tflops"], "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": r8["ms_per_step"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d,
                   "causal": w.causal, "input_dtype": w.dtype, "parallelism": f"replicas{world}",
                   "l2": "inputs larger than L2 (q, k, v = %.0f MB per rank)" % (3 * q.numel() * 2 / 1e6)},
        "modes": {
            "int8_qk": {"tflops": r8["tflops"], "ms_per_step": r8["ms_per_step"],
                        "prepass_ms": r8["kernel_ms"][0], "fused_ms": fused_ms,
                        "fused_tflops": achieved,
                        "prepass_gbs": _prepass_bytes(w) / (r8["kernel_ms"][0] * 1e-3) / 1e9,
                        "prepass_frac_of_hbm_peak": _prepass_bytes(w) / (r8["kernel_ms"][0] * 1e-3) / 1e9
                        / peaks["hbm_gbs"]},
            "fp8_qk": {"tflops": rf["tflops"], "ms_per_step": rf["ms_per_step"],
                       "prepass_ms": rf["kernel_ms"][0], "fused_ms": rf["kernel_ms"][1],
                       "fused_tflops": flops / (rf["kernel_ms"][1] * 1e-3) / 1e12,
                       "frac_of_mixed_peak": (flops / (rf["kernel_ms"][1] * 1e-3) / 1e12) / mixed_peak},
            "bf16_exact": {"tflops": rb["tflops"], "ms_per_step": rb["ms_per_step"],
                           "frac_of_bf16_peak": (flops / (rb["kernel_ms"][0] * 1e-3) / 1e12) / bf16_peak,
                           "traffic": _measured_traffic("bf16_exact"),
                           "algorithmic_bytes": _fused_bytes(w, "bf16_exact")},
        },
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": mixed_peak, "unit": "TFLOP/s",
                     "frac": achieved / mixed_peak, "traffic": _measured_traffic("int8_qk"),
                     "algorithmic_bytes": _fused_bytes(w, "int8_qk"),
                     "kernel": "attn_fwd_kernel<128,int8,bf16>",
                     "peak_note": ("4/3 x measured bf16 %s (%s): INT8 half of the FLOPs at 2x the bf16 rate"
                                   % ("sustained" if long_region else "burst", peaks["source"]))},
        "gpu_launches": 4 * args.steps,
        "clocks": clocks,
    }
    if e2e:
        line["e2e"] = e2e
    if not args.no_decode:
        line["decode"] = run_decode(args, dev, world, peaks)
        line["prefix_mask"] = run_prefix_mask(args, dev, world, peaks)
        line["context_parallel"] = run_context_parallel(args, dev, world, peaks)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    return line


def run_decode(args, dev, world, peaks):
    """KV-cache decode (attn_decode) on the named decode workloads: device time of back-to-back
    calls (every call reads its whole cache, 0.18-2.1 GB, larger than L2), bandwidth over the
    algorithmic bytes (used K and V once, q and o), against the measured HBM copy bandwidth."""
    import tiled_attention_22_b200 as ta

    out = {}
    for cfg, w in DECODE_WORKLOADS.items():
        q, k, v, lens = make_decode_inputs(w)
        q, k, v, lens_d = q.to(dev), k.to(dev), v.to(dev), lens.to(dev)
        ws = torch.zeros(ta.attn_decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, 0), device=dev,
                         dtype=torch.uint8)
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.Hq, w.Nq), device=dev, dtype=torch.float32)

        def call():
            ta.attn_decode(q, k, v, lens_d, causal=w.causal, scale=w.scale, out=o, lse=lse, workspace=ws)

        for _ in range(max(3, args.warmup)):
            call()
        torch.cuda.synchronize()
        _barrier(world)
        n = 50
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n):
            call()
        e1.record()
        torch.cuda.synchronize()
        _barrier(world)
        ms = _max_over_ranks(e0.elapsed_time(e1), world, dev) / n
        if ta.attn_check_status() != 0:
            raise RuntimeError("device-side wait timed out in the decode benchmark")
        nbytes = decode_bytes(w.B, w.Hq, w.Hkv, w.Nq, w.d, lens.tolist())
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[w.name] = {"ms_per_call": ms, "GB/s": gbs * world, "frac_of_hbm_peak": gbs / peaks["hbm_gbs"],
                       "bytes_per_call": nbytes, "calls": n, "kernel": "attn_decode_kernel<16,bf16>",
                       "launches_per_call": 1}
        del q, k, v, o, ws
        torch.cuda.empty_cache()
    out["peak_note"] = "HBM copy bandwidth %.0f GB/s (%s)" % (peaks["hbm_gbs"], peaks["source"])
    return out


def run_prefix_mask(args, dev, world, peaks):
    """Row-prefix-masked forward (attn_fwd_prefix_masked) on the APB-shaped workload: device time
    of back-to-back calls (inputs larger than L2), TFLOP/s over the visible (query, key) pairs
    (4 d FLOPs each), against the measured bf16 GEMM rate."""
    import tiled_attention_22_b200 as ta

    out = {}
    for cfg, w in APB_WORKLOADS.items():
        q, k, v = (t.to(dev) for t in make_apb_inputs(w))
        lim = ta.apb_row_limits(w.anchor, w.passing, w.local, device=dev)
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.Hq, w.Nq), device=dev, dtype=torch.float32)
        flops = 4.0 * w.B * w.Hq * w.d * float(lim.clamp(0, w.Nk).sum().item())

        def call():
            ta.attn_fwd_prefix_masked(q, k, v, lim, scale=w.scale, out=o, lse=lse)

        for _ in range(max(3, args.warmup)):
            call()
        torch.cuda.synchronize()
        _barrier(world)
        n = 20
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n):
            call()
        e1.record()
        torch.cuda.synchronize()
        _barrier(world)
        ms = _max_over_ranks(e0.elapsed_time(e1), world, dev) / n
        if ta.attn_check_status() != 0:
            raise RuntimeError("device-side wait timed out in the prefix-mask benchmark")
        tf = flops / (ms * 1e-3) / 1e12
        out[w.name] = {"ms_per_call": ms, "TFLOP/s": tf * world, "frac_of_bf16_peak": tf / peaks["bf16"],
                       "flops_per_call": flops, "calls": n, "kernel": "attn_fwd_kernel<128,bf16>",
                       "launches_per_call": 1}
        del q, k, v, o
        torch.cuda.empty_cache()
    out["peak_note"] = "bf16 dense GEMM %.0f TFLOP/s (%s, burst)" % (peaks["bf16"], peaks["source"])
    return out


def run_context_parallel(args, dev, world, peaks, ranks=4):
    """Context-parallel (ring) attention on the 131K-token GQA workload split over ``ranks`` ranks,
    emulated on this GPU: each rank's steps (fused kernel + lse merge per visible key block) run
    back to back with the blocks already split; no exchange (its NVLink cost is not measured).
    Reported beside one fused-kernel call over the whole sequence, both in bf16_exact."""
    import tiled_attention_22_b200 as ta
    from tiled_attention_22_b200.ring import ring_rank_emulated, ring_schedule

    w = WORKLOADS[5]
    q, k, v = (t.to(dev) for t in make_inputs(w))
    n = w.N // ranks
    qs = [q[:, :, r * n:(r + 1) * n].contiguous() for r in range(ranks)]
    kv = [(k[:, :, j * n:(j + 1) * n].contiguous(), v[:, :, j * n:(j + 1) * n].contiguous()) for j in range(ranks)]
    flops = w.flops()

    def ring():
        for r in range(ranks):
            ring_rank_emulated(qs[r], kv, r, causal=w.causal, scale=w.scale)

    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.N), device=dev, dtype=torch.float32)

    def whole():
        ta.attn_fwd(q, k, v, causal=w.causal, scale=w.scale, out=o, lse=lse)

    res = {}
    for name, fn in (("ring", ring), ("single_call", whole)):
        fn()
        torch.cuda.synchronize()
        _barrier(world)
        n_calls = 3
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n_calls):
            fn()
        e1.record()
        torch.cuda.synchronize()
        _barrier(world)
        res[name] = _max_over_ranks(e0.elapsed_time(e1), world, dev) / n_calls
    if ta.attn_check_status() != 0:
        raise RuntimeError("device-side wait timed out in the context-parallel benchmark")
    steps = sum(kind != "skip" for r in range(ranks) for _, _, kind in ring_schedule(r, ranks, w.causal))
    tf = flops / (res["ring"] * 1e-3) / 1e12
    out = {w.name + f"_ring{ranks}": {
        "ms_per_call": res["ring"], "TFLOP/s": tf * world, "frac_of_bf16_peak": tf / peaks["bf16_sustained"],
        "single_call_ms": res["single_call"], "ring_over_single": res["ring"] / res["single_call"],
        "launches_per_call": 2 * steps, "kernels": "attn_fwd_persistent_kernel<128,bf16> + lse_merge_kernel<128,bf16>",
        "note": "all ranks' steps on one GPU; the key/value exchange over NVLink is not timed"}}
    out["peak_note"] = "bf16 dense GEMM %.0f TFLOP/s (%s, sustained)" % (peaks["bf16_sustained"], peaks["source"])
    del q, k, v, qs, kv, o
    torch.cuda.empty_cache()
    return out


def _fused_bytes(w, mode):
    """Algorithmic bytes of one fused-kernel launch: Q and K read once (1 B/elt as INT8 codes,
    2 B/elt in bf16_exact), V read once, O written once, lse written (4 B/row); scales and the
    lse bias are per block / per row."""
    nq = w.B * w.Hq * w.N * w.d
    nk = w.B * w.Hkv * w.N * w.d
    qk = 1 if mode == "int8_qk" else 2
    extra = 4 * w.B * w.Hq * w.N * (2 if mode == "int8_qk" else 1)  # lse (+ bias)
    return qk * nq + qk * nk + 2 * nk + 2 * nq + extra


def _prepass_bytes(w):
    """Algorithmic bytes of the pre-pass: K and Q each read once in 16-bit and written once as 8-bit
    codes, plus the lse bias (4 B per query row); scales and the mean are small."""
    nk = w.B * w.Hkv * w.N * w.d
    nq = w.B * w.Hq * w.N * w.d
    return 3 * nk + 3 * nq + 4 * w.B * w.Hq * w.N


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--config", type=int, default=2)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true", help="skip the measurements of the other paths (KV-cache decode, prefix mask, ring)")
    ap.add_argument("--modes", default="int8_qk,bf16_exact,fp8_qk",
                    help="modes to time (the headline value is int8_qk; drop one only for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = WORKLOADS[args.config]
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        line = run_reference(args, w, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    world, rank, local = _dist_setup(args.gpus)
    try:
        line = run_native(args, w, world, rank, local)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
