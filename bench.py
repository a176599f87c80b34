#!/usr/bin/env python
"""Benchmark of one sparse MoE FFN layer (Step 3.5 Flash shape) on B200 through libstepmoe.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode|prefill|skewed|mtp|tiny]
                    [--impl ours|reference]

A step is one pass of the whole layer (route -> permute -> expert FFNs -> combine, one
smoe_forward call) over one batch of seeded synthetic tokens, weights resident in HBM. The
default workload is the decode batch (T=64, hidden 4096, 288 experts top-8, intermediate 1280,
one shared expert). Prints one JSON line on rank 0.

Multi-GPU: the layer does not shard across GPUs here (no exchange step), so N GPUs run N
independent replicas of the same workload, launched one process per GPU by torchrun; the
timed region is bracketed by barriers and the slowest rank's time is reported (value = all
ranks' tokens / that time).

--impl reference times the CPU fp64 oracle as it stands on the host cores, on a bounded
sample of the same workload (there is no other reference implementation of this layer).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

REPO = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, REPO)

METRIC = "MoE-layer tokens/s at 1 B200; achieved HBM GB/s (decode) / TFLOPS (prefill)"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024


# ------------------------------------------------------------------------------------ helpers
def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--workload", default="decode")
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-sample-tokens", type=int, default=4)
    p.add_argument("--cpu-seconds", type=float, default=10.0)
    p.add_argument("--diag", action="store_true", help="time smoe_forward_diag (layer + monitoring outputs)")
    p.add_argument("--fp8", action="store_true", help="time smoe_forward_fp8 (e4m3 experts, per-row scales)")
    return p.parse_args(argv)


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), int(os.environ.get("WORLD_SIZE", 1))


def init_dist(world: int, backend: str):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))


def max_over_ranks(v: float, device=None) -> float:
    """Max of a float over all ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def measured_peaks():
    path = os.path.join(REPO, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def source_sha(paths) -> str:
    """Hash of the code of the given sources with comments and whitespace removed, so that an
    edit of comments alone keeps the committed counters valid."""
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(REPO, p), encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


GEMM_SOURCES = ["sparse_moe_layer_smoe_b200/csrc/expert_ffn.cu", "sparse_moe_layer_smoe_b200/csrc/common.cuh"]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the current source."""
    path = os.path.join(REPO, "profiles", f"{kernel}_{workload}_traffic.txt")
    if not os.path.exists(path):
        return None
    kv = {}
    with open(path) as f:
        for line in f:
            if ":" in line:
                a, b = line.split(":", 1)
                kv[a.strip()] = b.strip()
    if kv.get("source_sha") != source_sha(GEMM_SOURCES):
        return None
    try:
        return float(kv["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """Samples the SM clock and clock-event reasons with NVML while the timed region runs."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.005):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self.period = period_s
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ------------------------------------------------------------------------------------ CPU oracle leg
def oracle_sample(w, n_tokens: int):
    """Inputs of the oracle for the first n_tokens tokens: fp64 x, router, bias and fp64 weights of
    every expert those tokens select (prepared before any timing)."""
    import numpy as np

    import oracle
    import synth
    rows = np.arange(min(n_tokens, w.T))
    x64 = oracle.bf16_to_f64(synth.host_x_rows(w, rows))
    wr64 = oracle.f32_to_f64(synth.host_w_router(w))
    bias = synth.host_bias(w).astype(np.float64)
    r = oracle.route(x64, wr64, bias, w.k, w.route_scale)
    need = sorted(set(r.idx.reshape(-1).tolist())) + [w.E]
    experts = {e: tuple(oracle.bf16_to_f64(a) for a in synth.host_expert(w, e)) for e in need}
    return x64, wr64, bias, experts


def oracle_step(w, x64, wr64, bias, experts):
    import oracle
    r = oracle.route(x64, wr64, bias, w.k, w.route_scale)
    return oracle.moe_sparse(x64, r, lambda e: experts[e], w.E)


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_baseline(w, n_tokens: int, min_seconds: float):
    x64, wr64, bias, experts = oracle_sample(w, n_tokens)
    oracle_step(w, x64, wr64, bias, experts)   # warm-up
    done, t0 = 0, time.perf_counter()
    while True:
        oracle_step(w, x64, wr64, bias, experts)
        done += x64.shape[0]
        el = time.perf_counter() - t0
        if el >= min_seconds:
            break
    return {"value": done / el, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"first {x64.shape[0]} tokens of the {w.name} batch (fp64 numpy oracle, sparse mode; fp64 "
                      f"weights of their {len(experts)} experts prepared untimed), repeated for {el:.1f} s"}


def run_reference(args):
    import synth
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    w = synth.WORKLOADS[args.workload]
    x64, wr64, bias, experts = oracle_sample(w, args.cpu_sample_tokens)
    n = x64.shape[0]
    for i in range(args.warmup):
        oracle_step(w, x64[i % n:i % n + 1], wr64, bias, experts)
    t0 = time.perf_counter()
    for i in range(args.steps):
        oracle_step(w, x64[i % n:i % n + 1], wr64, bias, experts)
    el = time.perf_counter() - t0
    value = args.steps / el
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": f"one token per step, cycling over the first {n} tokens of the {w.name} "
                                       f"batch; fp64 weights of their {len(experts)} experts prepared untimed"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------------ GPU leg
def workload_config(w):
    return {"workload": w.name, "T": w.T, "hidden": w.H, "experts": w.E, "top_k": w.k, "inter": w.I,
            "shared_inter": w.Is, "route_scale": w.route_scale, "bias": w.bias, "spike_rows": w.spike_rows,
            "swiglu_limit": w.swiglu_limit, "swiglu_limit_shared": w.swiglu_limit_shared,
            "parallelism": "replicas",
            "l2": "inputs larger than L2: every step streams the active experts' bf16 weights (GBs) from HBM"}


def run_ours(args):
    import torch

    import sparse_moe_layer_smoe_b200 as smoe
    import synth

    rank, local, world = dist_env()
    torch.cuda.set_device(local)
    init_dist(world, "nccl")
    dev = torch.device("cuda", local)
    w = synth.WORKLOADS[args.workload]
    cfg = smoe.config(w.H, w.E, w.k, w.I, w.Is, w.route_scale, w.swiglu_limit, w.swiglu_limit_shared)
    T = w.T

    x = synth.dev_x(w, device=dev)
    wr, bias = synth.dev_router(w, device=dev)
    experts = synth.dev_experts(w, device=dev)
    packed = smoe.pack_weights_fp8(cfg, *experts) if args.fp8 else smoe.pack_weights(cfg, *experts)
    torch.cuda.synchronize()
    del experts
    torch.cuda.empty_cache()
    ws = smoe.workspace(cfg, T, device=dev, fp8=args.fp8)
    out = torch.empty(T, w.H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()
    diag = smoe.diag_buffers(cfg, T, device=dev) if args.diag else None

    def forward(x_):
        if args.fp8:
            smoe.smoe_forward_fp8(cfg, x_, T, wr, bias, packed, out, ws)
        elif diag is None:
            smoe.smoe_forward(cfg, x_, T, wr, bias, packed, out, ws)
        else:
            smoe.smoe_forward_diag(cfg, x_, T, wr, bias, packed, out, diag, ws)

    # routing statistics of this batch (for the algorithmic byte count): experts touched
    idx = torch.empty(T, w.k, dtype=torch.int32, device=dev)
    wt = torch.empty(T, w.k, dtype=torch.float32, device=dev)
    sws = smoe.workspace(cfg, T, forward=False, device=dev)
    smoe.smoe_route(cfg, x, T, wr, bias, idx, wt, None, sws)
    counts = torch.bincount(idx.view(-1).long(), minlength=w.E)
    touched = int((counts > 0).sum().item())
    del sws

    # ---- device-resident timing (value)
    for _ in range(args.warmup):
        forward(x)
    torch.cuda.synchronize()
    launches_per_step = smoe.smoe_last_launch_count()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        ev0.record(stream)
        for _ in range(args.steps):
            forward(x)
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier()
    ms = ev0.elapsed_time(ev1) / args.steps
    ms = max_over_ranks(ms, dev)

    # ---- per-kernel split, in a separate pass: the library records CUDA events around each of
    # its launches, which serialises the kernels (the timed steps above let each kernel launch
    # while its predecessor finishes)
    ksteps = min(args.steps, 20)
    smoe.smoe_timing_begin(ksteps * launches_per_step + 16)
    for _ in range(ksteps):
        forward(x)
    torch.cuda.synchronize()
    ktimes = smoe.smoe_timing_end()
    err = smoe.smoe_get_device_error(ws)
    if err != 0:
        raise RuntimeError(f"device error word {smoe.STATUS.get(err, err)}")

    # ---- end to end through the C-ABI from pinned host buffers (copies inside the region)
    x_host = x.cpu().pin_memory()
    out_host = torch.empty(T, w.H, dtype=torch.bfloat16).pin_memory()
    x_in = torch.empty_like(x)

    def e2e_step():
        x_in.copy_(x_host, non_blocking=True)
        forward(x_in)
        out_host.copy_(out, non_blocking=True)
        stream.synchronize()

    for _ in range(args.warmup):
        e2e_step()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, dev)

    # ---- roofline of the dominant kernel
    peaks, peak_src = measured_peaks()
    dom = max(ktimes.items(), key=lambda kv: kv[1][1])[0] if ktimes else None
    H, I, E, k = w.H, w.I, w.E, w.k
    wb = 1 if args.fp8 else 2   # bytes per weight (e4m3 or bf16); e4m3 adds one fp32 scale per weight row
    ab = 1 if args.fp8 else 2   # bytes per GEMM input activation
    gate_up_bytes = (touched + 1) * 2 * I * (H * wb + (4 if args.fp8 else 0)) + (T * k + T) * H * ab + (T * k + T) * I * 2
    down_bytes = (touched + 1) * H * (I * wb + (4 if args.fp8 else 0)) + (T * k + T) * I * ab + (T * k + T) * H * 2
    kern_bytes = {"expert_gateup": gate_up_bytes, "expert_down": down_bytes}
    kern_flops = {"expert_gateup": 2.0 * (T * k + T) * 2 * I * H, "expert_down": 2.0 * (T * k + T) * H * I}
    roof = None
    if dom in kern_bytes:
        launches, tot = ktimes[dom]
        avg_s = tot / launches / 1e3
        intensity = kern_flops[dom] / kern_bytes[dom]
        # the tensor peak of the contraction's own dtype: e4m3 = the measured bf16 peak x 2, the
        # nominal dense ratio (4.5 / 2.25 PFLOP/s)
        tc_peak = peaks["bf16_tflops_sustained"] * (2.0 if args.fp8 else 1.0)
        tc_src = ("MEASURED_PEAKS.json bf16_tflops_sustained x 2 (nominal e4m3 / bf16 ratio)" if args.fp8
                  else "MEASURED_PEAKS.json bf16_tflops_sustained")
        ridge = tc_peak * 1e12 / (peaks["hbm_gbs"] * 1e9)
        traffic = profiled_traffic(dom, w.name + ("_fp8" if args.fp8 else ""))
        if intensity < ridge:
            ach = kern_bytes[dom] / avg_s / 1e9
            roof = {"bound": "hbm", "kernel": dom, "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": ach / peaks["hbm_gbs"], "traffic": traffic,
                    "algorithmic_bytes": kern_bytes[dom], "avg_launch_ms": avg_s * 1e3,
                    "peak_source": f"MEASURED_PEAKS.json hbm_gbs ({peak_src})"}
        else:
            ach = kern_flops[dom] / avg_s / 1e12
            roof = {"bound": "tensor", "kernel": dom, "achieved": ach, "peak": tc_peak,
                    "unit": "TFLOP/s", "frac": ach / tc_peak, "traffic": traffic, "algorithmic_flops": kern_flops[dom],
                    "avg_launch_ms": avg_s * 1e3, "peak_source": f"{tc_src} ({peak_src})"}
    layer_bytes = (touched + 1) * 3 * H * I * wb + E * H * 4 + 2 * T * H * 2
    layer_flops = 2.0 * T * (k + 1) * 3 * H * I

    line = {"metric": METRIC, "value": world * T / (ms / 1e3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3" if args.fp8 else "bf16", "data": "synthetic",
            "config": {**workload_config(w), **({"diag": True} if args.diag else {}),
                       **({"experts": "e4m3, per-row fp32 scales; router fp32"} if args.fp8 else {})},
            "layer": {"hbm_gbs": layer_bytes / (ms / 1e3) / 1e9, "tflops": layer_flops / (ms / 1e3) / 1e12,
                      "experts_touched": touched, "algorithmic_bytes": layer_bytes},
            "kernels_ms_per_step": {n: t / ksteps for n, (_, t) in sorted(ktimes.items(), key=lambda kv: -kv[1][1])},
            "roofline": roof,
            "e2e": {"value": world * T / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": T * H * 2,
                    "d2h_bytes_per_step": T * H * 2, "ms_per_step": e2e_ms},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk.summary()}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_sample_tokens, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
