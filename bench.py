#!/usr/bin/env python
"""Benchmark of one sparse MoE FFN layer (Step 3.5 Flash shape) on B200 through libstepmoe.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode|prefill|skewed|mtp|tiny]
                    [--impl ours|reference]

A step is one pass of the whole layer (route -> permute -> expert FFNs -> combine, one
smoe_forward call) over one batch of seeded synthetic tokens, weights resident in HBM. The
headline workload is the decode batch (T=64, hidden 4096, 288 experts top-8, intermediate 1280,
one shared expert); the same run also times the prefill (T=8192), skewed (T=4096, Zipf
popularity, 16 dead experts) and MTP-verify (T=512, activation spikes) batches on the same
weights and reports each under "workloads" with its own roofline, step-time spread, expert
statistics and routing check. Prints one JSON line on rank 0.

Multi-GPU: the layer does not shard across GPUs here (no exchange step), so N GPUs run N
independent replicas of the same workload, launched one process per GPU by torchrun; the
timed region is bracketed by barriers and the slowest rank's time is reported (value = all
ranks' tokens / that time).

--impl reference times the C++ fp64 oracle as it stands on the host cores, on a bounded
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
    p.add_argument("--workload", default="decode", help="the headline workload (value, e2e, roofline)")
    p.add_argument("--workloads", default="decode,prefill,skewed,mtp",
                   help="comma list of further workloads of the same layer shape timed in the same run and "
                        "reported under 'workloads' ('none': the headline only)")
    p.add_argument("--pct-steps", type=int, default=50, help="steps of the per-step spread pass (p10/p50/p90)")
    p.add_argument("--cooldown", type=float, default=2.0,
                   help="idle seconds before each workload after the headline, so that each one starts from the "
                        "same power state instead of inheriting the previous workload's")
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

    def __init__(self, index: int, period_s: float = 0.001):
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
# The oracle (the C++ fp64 program, test infrastructure) is run here only: timed as the CPU
# baseline and the reference arm, and used untimed to count near-tie tokens and to check the
# GPU's selections against its fp64 router.
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


def oracle_forward_seconds(w, x64, wr64, bias, experts, repeats: int) -> float:
    """Seconds of `repeats` oracle passes (route + sparse layer) over x64, timed inside the C++
    oracle with std::chrono::steady_clock."""
    import oracle
    _, sec = oracle.cpp.forward_timed(x64, wr64, bias, w.k, w.route_scale, lambda e: experts[e], w.E, repeats,
                                      w.swiglu_limit, w.swiglu_limit_shared)
    return sec


def oracle_threads() -> int:
    import oracle
    return oracle.cpp.threads()


def cpu_baseline(w, n_tokens: int, min_seconds: float):
    x64, wr64, bias, experts = oracle_sample(w, n_tokens)
    one = oracle_forward_seconds(w, x64, wr64, bias, experts, 1)   # also the warm-up
    repeats = max(1, int(min_seconds / max(one, 1e-6)))
    el = oracle_forward_seconds(w, x64, wr64, bias, experts, repeats)
    done = repeats * x64.shape[0]
    return {"value": done / el, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
            "implementation": "C++17 fp64 oracle (oracle/smoe_oracle.cpp: plain loops, std::sort, std::thread)",
            "sample": f"first {x64.shape[0]} tokens of the {w.name} batch, {repeats} passes of route + sparse layer "
                      f"timed with std::chrono in the C++ oracle ({el:.1f} s); fp64 weights of their "
                      f"{len(experts)} experts prepared untimed"}


def routing_check(w, gpu_idx):
    """The GPU's selections against the oracle's fp64 router on the whole batch (untimed):
    near-tie tokens (8th/9th biased-score gap < 1e-5), selections that differ outside near ties
    (must be 0), and tokens whose selected order differs from the oracle's — within the 1e-5
    band, where fp32 rounding may swap two experts, and beyond it (must be 0)."""
    import numpy as np

    import oracle
    import synth
    r = oracle.route(oracle.bf16_to_f64(synth.host_x(w)), oracle.f32_to_f64(synth.host_w_router(w)),
                     synth.host_bias(w).astype(np.float64), w.k, w.route_scale)
    near = r.near_tie
    differs = np.array([set(a) != set(b) for a, b in zip(gpu_idx.tolist(), r.idx.tolist())])
    order_in_band = order_beyond = 0
    for t in np.nonzero(~differs & ~near)[0]:
        g = gpu_idx[t]
        if np.array_equal(g, r.idx[t]):
            continue
        b = r.bhat[t, g]
        if np.all(b[:-1] >= b[1:] - oracle.NEAR_TIE_EPS):
            order_in_band += 1
        else:
            order_beyond += 1
    return {"near_tie_tokens": int(near.sum()), "selection_differs_outside_near_ties": int((differs & ~near).sum()),
            "selection_differs_at_near_ties": int((differs & near).sum()),
            "order_differs_within_1e-5": int(order_in_band), "order_differs_beyond_1e-5": int(order_beyond),
            "oracle": "C++ fp64 router"}


def run_reference(args):
    import synth
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    w = synth.WORKLOADS[args.workload]
    x64, wr64, bias, experts = oracle_sample(w, args.cpu_sample_tokens)
    n = x64.shape[0]
    for i in range(args.warmup):
        oracle_forward_seconds(w, x64[i % n:i % n + 1], wr64, bias, experts, 1)
    el = 0.0
    for i in range(args.steps):
        el += oracle_forward_seconds(w, x64[i % n:i % n + 1], wr64, bias, experts, 1)
    value = args.steps / el
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
                             "implementation": "C++17 fp64 oracle (oracle/smoe_oracle.cpp: plain loops, std::sort, "
                                               "std::thread)",
                             "sample": f"one token per step, cycling over the first {n} tokens of the {w.name} "
                                       f"batch, each step timed with std::chrono in the C++ oracle; fp64 weights "
                                       f"of their {len(experts)} experts prepared untimed"},
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


def percentiles(v):
    import numpy as np
    a = np.asarray(v, dtype=np.float64)
    return {"p10": float(np.percentile(a, 10)), "p50": float(np.percentile(a, 50)),
            "p90": float(np.percentile(a, 90)), "steps": int(a.size)}


def kernel_bytes_flops(w, touched: int, fp8: bool):
    """Algorithmic bytes and flops of one launch of each expert GEMM: the weights of the touched
    experts and the shared one, the GEMM's input activations and its output."""
    H, I, T, k = w.H, w.I, w.T, w.k
    wb = 1 if fp8 else 2   # bytes per weight (e4m3 or bf16); e4m3 adds one fp32 scale per weight row
    ab = 1 if fp8 else 2   # bytes per GEMM input activation
    rows = T * k + T
    gate_up = (touched + 1) * 2 * I * (H * wb + (4 if fp8 else 0)) + rows * H * ab + rows * I * 2
    down = (touched + 1) * H * (I * wb + (4 if fp8 else 0)) + rows * I * ab + rows * H * 2
    return ({"expert_gateup": gate_up, "expert_down": down},
            {"expert_gateup": 2.0 * rows * 2 * I * H, "expert_down": 2.0 * rows * H * I})


def measure(smoe, w, packed, args, dev, headline: bool):
    """Time one workload: the device-resident steps (value), per-kernel split, per-step spread and
    the end-to-end steps from pinned host buffers. Returns (entry, GPU top-k indices)."""
    import torch

    import synth
    fp8 = args.fp8
    cfg = smoe.config(w.H, w.E, w.k, w.I, w.Is, w.route_scale, w.swiglu_limit, w.swiglu_limit_shared)
    T, E = w.T, w.E
    rank, local, world = dist_env()
    x = synth.dev_x(w, device=dev)
    wr, bias = synth.dev_router(w, device=dev)
    ws = smoe.workspace(cfg, T, device=dev, fp8=fp8)
    out = torch.empty(T, w.H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()
    diag = smoe.diag_buffers(cfg, T, device=dev) if args.diag else None

    def forward(x_):
        if fp8:
            smoe.smoe_forward_fp8(cfg, x_, T, wr, bias, packed, out, ws)
        elif diag is None:
            smoe.smoe_forward(cfg, x_, T, wr, bias, packed, out, ws)
        else:
            smoe.smoe_forward_diag(cfg, x_, T, wr, bias, packed, out, diag, ws)

    # routing of this batch on the GPU (for the algorithmic byte count and the expert statistics)
    idx = torch.empty(T, w.k, dtype=torch.int32, device=dev)
    wt = torch.empty(T, w.k, dtype=torch.float32, device=dev)
    sws = smoe.workspace(cfg, T, forward=False, device=dev)
    smoe.smoe_route(cfg, x, T, wr, bias, idx, wt, None, sws)
    counts = torch.bincount(idx.view(-1).long(), minlength=E).cpu()
    gpu_idx = idx.cpu().numpy()
    del sws
    touched = int((counts > 0).sum().item())
    live = counts[counts > 0]
    experts = {"touched": touched, "dead": E - touched, "max_count": int(counts.max().item()),
               "min_count_live": int(live.min().item()) if touched else 0, "mean_count": T * w.k / E}

    # ---- device-resident timing (value)
    if not headline and args.cooldown > 0:
        # the 1 kW power cap lowers the clock after a tensor-heavy workload for a while: idle first
        torch.cuda.synchronize()
        time.sleep(args.cooldown)
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
    ms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps, dev)

    # ---- per-step spread, in a pass of its own: an event between steps keeps the next step's
    # first kernel from starting under the previous step's last one
    n_pct = max(args.steps, args.pct_steps)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n_pct + 1)]
    evs[0].record(stream)
    for i in range(n_pct):
        forward(x)
        evs[i + 1].record(stream)
    torch.cuda.synchronize()
    spread = percentiles([evs[i].elapsed_time(evs[i + 1]) for i in range(n_pct)])

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
        raise RuntimeError(f"{w.name}: device error word {smoe.STATUS.get(err, err)}")

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

    # ---- rooflines: the layer, and its dominant kernel
    peaks, peak_src = measured_peaks()
    tc_mult = 2.0 if fp8 else 1.0   # e4m3 peak = the measured bf16 peak x 2 (nominal 4.5 / 2.25 PFLOP/s)
    tc_sus, tc_burst = peaks["bf16_tflops_sustained"] * tc_mult, peaks["bf16_tflops"] * tc_mult
    H, I, k = w.H, w.I, w.k
    wb = 1 if fp8 else 2
    layer_bytes = (touched + 1) * 3 * H * I * wb + E * H * 4 + 2 * T * H * 2
    layer_flops = 2.0 * T * (k + 1) * 3 * H * I
    s = ms / 1e3
    layer = {"hbm_gbs": layer_bytes / s / 1e9, "hbm_frac": layer_bytes / s / 1e9 / peaks["hbm_gbs"],
             "tflops": layer_flops / s / 1e12, "tflops_frac_sustained": layer_flops / s / 1e12 / tc_sus,
             "tflops_frac_burst": layer_flops / s / 1e12 / tc_burst, "algorithmic_bytes": layer_bytes,
             "algorithmic_flops": layer_flops,
             "bound": "hbm" if layer_bytes / (peaks["hbm_gbs"] * 1e9) >= layer_flops / (tc_sus * 1e12) else "tensor"}
    kern_bytes, kern_flops = kernel_bytes_flops(w, touched, fp8)
    dom = max(ktimes.items(), key=lambda kv: kv[1][1])[0] if ktimes else None
    roof = None
    if dom in kern_bytes:
        launches, tot = ktimes[dom]
        avg_s = tot / launches / 1e3
        hbm_ach = kern_bytes[dom] / avg_s / 1e9
        tc_ach = kern_flops[dom] / avg_s / 1e12
        t_hbm = kern_bytes[dom] / (peaks["hbm_gbs"] * 1e9)
        t_tc = kern_flops[dom] / (tc_sus * 1e12)
        traffic = profiled_traffic(dom, w.name + ("_fp8" if fp8 else ""))
        common = {"kernel": dom, "traffic": traffic, "algorithmic_bytes": kern_bytes[dom],
                  "algorithmic_flops": kern_flops[dom], "avg_launch_ms": avg_s * 1e3,
                  "hbm_gbs": hbm_ach, "hbm_frac": hbm_ach / peaks["hbm_gbs"], "tflops": tc_ach,
                  "tflops_frac_sustained": tc_ach / tc_sus, "tflops_frac_burst": tc_ach / tc_burst}
        tc_name = "bf16_tflops{}" + (" x 2 (nominal e4m3 / bf16 ratio)" if fp8 else "")
        if t_hbm >= t_tc:
            roof = {"bound": "hbm", "achieved": hbm_ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": hbm_ach / peaks["hbm_gbs"], **common,
                    "peak_source": f"MEASURED_PEAKS.json hbm_gbs ({peak_src})"}
        else:
            roof = {"bound": "tensor", "achieved": tc_ach, "peak": tc_sus, "unit": "TFLOP/s",
                    "frac": tc_ach / tc_sus, **common,
                    "peak_source": f"MEASURED_PEAKS.json {tc_name.format('_sustained')} ({peak_src}); the burst "
                                   f"peak {tc_burst:.1f} gives tflops_frac_burst"}

    entry = {"value": world * T / s, "unit": UNIT, "ms_per_step": ms, "step_ms": spread,
             "config": {**workload_config(w), **({"diag": True} if args.diag else {}),
                        **({"experts": "e4m3, per-row fp32 scales; router fp32"} if fp8 else {})},
             "layer": layer, "experts": experts,
             "kernels_ms_per_step": {n: t / ksteps for n, (_, t) in sorted(ktimes.items(), key=lambda kv: -kv[1][1])},
             "roofline": roof,
             "e2e": {"value": world * T / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": T * H * 2,
                     "d2h_bytes_per_step": T * H * 2, "ms_per_step": e2e_ms},
             "gpu_launches": launches_per_step * args.steps, "launches_per_step": launches_per_step,
             "clocks": clk.summary()}
    del ws, x, out
    return entry, gpu_idx


def run_ours(args):
    import torch

    import sparse_moe_layer_smoe_b200 as smoe
    import synth

    rank, local, world = dist_env()
    torch.cuda.set_device(local)
    init_dist(world, "nccl")
    dev = torch.device("cuda", local)
    head = synth.WORKLOADS[args.workload]
    extra = [] if args.workloads in ("", "none") else [n for n in args.workloads.split(",") if n != head.name]
    for n in extra:
        if synth.WORKLOADS[n].H != head.H or synth.WORKLOADS[n].E != head.E or synth.WORKLOADS[n].I != head.I:
            raise SystemExit(f"--workloads: {n} has another layer shape than {head.name}")
    cfg = smoe.config(head.H, head.E, head.k, head.I, head.Is, head.route_scale)

    # the layer's weights, shared by every workload of this shape (same seed)
    experts = synth.dev_experts(head, device=dev)
    packed = smoe.pack_weights_fp8(cfg, *experts) if args.fp8 else smoe.pack_weights(cfg, *experts)
    torch.cuda.synchronize()
    del experts
    torch.cuda.empty_cache()

    results = {}
    for name in [head.name] + extra:
        results[name] = measure(smoe, synth.WORKLOADS[name], packed, args, dev, headline=(name == head.name))

    entry, _ = results[head.name]
    line = {"metric": METRIC, "value": entry["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": entry["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3" if args.fp8 else "bf16", "data": "synthetic",
            "config": entry["config"], "layer": entry["layer"], "experts": entry["experts"],
            "step_ms": entry["step_ms"], "kernels_ms_per_step": entry["kernels_ms_per_step"],
            "roofline": entry["roofline"], "e2e": entry["e2e"], "gpu_launches": entry["gpu_launches"],
            "clocks": entry["clocks"], "cooldown_s": args.cooldown,
            "workloads": {n: {kk: vv for kk, vv in e.items() if kk != "config"} | {"T": synth.WORKLOADS[n].T}
                          for n, (e, _) in results.items()}}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        for n, (e, gidx) in results.items():
            line["workloads"][n]["routing"] = routing_check(synth.WORKLOADS[n], gidx)
        line["routing"] = line["workloads"][head.name]["routing"]
        line["cpu_baseline"] = cpu_baseline(head, args.cpu_sample_tokens, args.cpu_seconds)
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
