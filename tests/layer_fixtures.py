"""Shared set-up for the GPU parity tests: device tensors from the seeded device generator,
host tensors for the oracle from the seeded host generator (bit-identical by construction and
checked in test_gpu_parity.py), and the parity tolerances.

Tolerances (from the layer's stated acceptance bar): relative Frobenius error <= 1e-2 and
per-element |err| <= 2e-2 * max|ref| for layer and FFN outputs; top-k indices bit-exact
except for near-tie tokens (8th/9th biased-score gap < 1e-5 in the fp64 oracle).
"""
from __future__ import annotations

import functools

import numpy as np

import oracle
import synth

REL_FRO = 1e-2
REL_MAX = 2e-2
STEP_WORKLOADS = ["decode", "prefill", "skewed", "mtp"]
ALL_WORKLOADS = ["tiny"] + STEP_WORKLOADS


def cfg_of(w: synth.Workload):
    import sparse_moe_layer_smoe_b200 as smoe
    return smoe.config(w.H, w.E, w.k, w.I, w.Is, w.route_scale, w.swiglu_limit, w.swiglu_limit_shared)


def limit_of(w: synth.Workload, g: int) -> float:
    """SwiGLU clamp limit of group g (g == E: the shared expert)."""
    return w.swiglu_limit_shared if g == w.E else w.swiglu_limit


def shape_key(w: synth.Workload):
    return (w.H, w.E, w.k, w.I, w.Is, w.seed, w.w_std)


@functools.lru_cache(maxsize=2)
def device_params(key):
    """Router weights and packed experts on cuda:0 for a layer shape (weights shared by workloads)."""
    import torch

    import sparse_moe_layer_smoe_b200 as smoe
    w = next(v for v in synth.WORKLOADS.values() if shape_key(v) == key)
    wr, _ = synth.dev_router(w)
    experts = synth.dev_experts(w)
    packed = smoe.pack_weights(cfg_of(w), *experts)
    torch.cuda.synchronize()
    del experts
    torch.cuda.empty_cache()
    return wr, packed


def device_inputs(name: str):
    import torch
    w = synth.WORKLOADS[name]
    wr, packed = device_params(shape_key(w))
    x = synth.dev_x(w)
    bias = torch.from_numpy(synth.host_bias(w)).cuda()
    return w, x, wr, bias, packed


@functools.lru_cache(maxsize=4)
def host_route(name: str) -> oracle.Route:
    w = synth.WORKLOADS[name]
    x = oracle.bf16_to_f64(synth.host_x(w))
    wr = oracle.f32_to_f64(synth.host_w_router(w))
    return oracle.route(x, wr, synth.host_bias(w).astype(np.float64), w.k, w.route_scale)


@functools.lru_cache(maxsize=2)
def host_x64(name: str) -> np.ndarray:
    return oracle.bf16_to_f64(synth.host_x(synth.WORKLOADS[name]))


class HostExperts:
    """fp64 expert weights generated on the host on demand (a small LRU of experts)."""

    def __init__(self, w: synth.Workload, cap: int = 24):
        self.w = w
        self.cap = cap
        self.cache: dict[int, tuple] = {}

    def __call__(self, e: int):
        if e not in self.cache:
            if len(self.cache) >= self.cap:
                self.cache.pop(next(iter(self.cache)))
            self.cache[e] = tuple(oracle.bf16_to_f64(a) for a in synth.host_expert(self.w, e))
        return self.cache[e]


def bf16_tensor_to_f64(t) -> np.ndarray:
    """Device bf16 tensor -> host fp64 (exact)."""
    import torch
    return oracle.bf16_to_f64(t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16))


def stratified_tokens(T: int, n: int, rng) -> list:
    """n tokens spread over the whole batch: one random token in each of n equal slices."""
    if T <= n:
        return list(range(T))
    edges = np.linspace(0, T, n + 1).astype(int)
    return [int(rng.integers(a, b)) for a, b in zip(edges[:-1], edges[1:]) if b > a]


def assert_close(gpu: np.ndarray, ref: np.ndarray, what: str, rel_fro=REL_FRO, rel_max=REL_MAX):
    err = gpu - ref
    fro = np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-300)
    mx = np.abs(err).max() / max(np.abs(ref).max(), 1e-300)
    assert fro <= rel_fro, f"{what}: relative Frobenius error {fro:.3e} > {rel_fro}"
    assert mx <= rel_max, f"{what}: max |err| / max|ref| = {mx:.3e} > {rel_max}"
    return fro, mx


def selection_ok(r: oracle.Route, t: int, gpu_set: tuple, k: int, max_enum: int = 14):
    """Whether the GPU's selected set is correct for token t, and the oracle set to compare with.

    Not near a tie: the set must equal the oracle's. Near a tie: the set must satisfy the band
    condition; when few experts sit in the band the oracle enumerates every valid set and the
    GPU's must be one of them."""
    ref = tuple(sorted(r.idx[t].tolist()))
    if not r.near_tie[t]:
        return gpu_set == ref, ref
    row = r.bhat[t]
    S = list(gpu_set)
    others = np.delete(row, S)
    valid = row[S].min() >= others.max() - oracle.NEAR_TIE_EPS
    v = np.sort(row)[::-1]
    band = int(np.sum(row >= v[k - 1] - oracle.NEAR_TIE_EPS))
    if band <= max_enum:
        return (gpu_set in oracle.valid_selections(row, k)) and valid, gpu_set
    return valid and gpu_set == ref, ref
