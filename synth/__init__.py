"""Seeded synthetic inputs for the sparse MoE FFN layer (shared by the oracle and the CUDA path).

This module holds none of the layer's arithmetic: no router, no top-k, no FFN. It
only produces the seeded tensors both sides are fed, and the workload recipes
(shapes, value distributions, bias pattern, spike rows) of the five layer
configurations. The counter-based generator is defined in ``synth_host.c``; the
host (C, OpenMP) and device (CUDA) implementations agree bit for bit, and
``normal_reference`` restates the definition in numpy so the C code can be
pinned on small sizes.

Workloads (Step 3.5 Flash model card, raw config fields ``hidden_size 4096``,
``moe_num_experts 288``, ``moe_top_k 8``, ``moe_intermediate_size 1280``,
``share_expert_dim 1280``, ``moe_router_scaling_factor 3``):

* ``tiny``     T=64,   H=512,  E=32,  k=4, I=Is=128, bias 0
* ``decode``   T=64,   Step shape, bias 0
* ``prefill``  T=8192, Step shape, bias 0
* ``skewed``   T=4096, Step shape, Zipf(1.2) popularity bias, 16 dead experts
* ``mtp``      T=512 (128 sequences x 4 tokens), 1% of rows (5) scaled x50
* ``mtp_clamp`` the MTP batch with the SwiGLU clamp of the deepest layers (routed 7, shared 16)

x ~ N(0, 1) -> bf16; router W_r ~ N(0, 0.02) fp32; expert weights ~ N(0, 0.02) -> bf16.
"""
from __future__ import annotations

import ctypes
import json
import math
import os
import struct
import subprocess
from dataclasses import dataclass, field

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
REPO = os.path.dirname(HERE)
HOST_LIB = os.path.join(HERE, "libsmoe_synth_host.so")
DEV_LIB = os.path.join(HERE, "libsmoe_synth_dev.so")

# standard deviation of c = 2*S - 8*65535 (S = sum of eight uniform 16-bit integers)
C_SD = math.sqrt(8.0 * (65536.0 ** 2 - 1.0) / 3.0)
G = 0x9E3779B97F4A7C15
M64 = (1 << 64) - 1

# tensor ids: distinct counters for each input tensor of a layer
TID_X, TID_WR, TID_WG, TID_WU, TID_WD, TID_WSG, TID_WSU, TID_WSD = 1, 2, 4, 5, 6, 7, 8, 9
TID_SPIKE_ROWS, TID_ZIPF_RANK = 10, 11


def scale_bits(std: float) -> int:
    """fp32 bit pattern of std / C_SD (the one multiplier both generators apply)."""
    return struct.unpack("<I", struct.pack("<f", std / C_SD))[0]


# ---------------------------------------------------------------------------------------------
# numpy restatement of the definition (slow; used to pin the C generator on small sizes)
# ---------------------------------------------------------------------------------------------
def _mix64_np(z: np.ndarray) -> np.ndarray:
    z = z.copy()
    with np.errstate(over="ignore"):
        z ^= z >> np.uint64(30)
        z *= np.uint64(0xBF58476D1CE4E5B9)
        z ^= z >> np.uint64(27)
        z *= np.uint64(0x94D049BB133111EB)
        z ^= z >> np.uint64(31)
    return z


def _key(seed: int, tid: int) -> int:
    z = np.array([(seed * G + tid) & M64], dtype=np.uint64)
    return int(_mix64_np(z)[0])


def normal_reference(n: int, seed: int, tid: int, std: float, index_base: int = 0) -> np.ndarray:
    """fp32 values z(index_base .. index_base+n-1) computed in numpy from the definition."""
    key = np.uint64(_key(seed, tid))
    i = np.arange(index_base, index_base + n, dtype=np.uint64)
    with np.errstate(over="ignore"):
        h0 = _mix64_np(key + (np.uint64(2) * i + np.uint64(1)) * np.uint64(G))
        h1 = _mix64_np(key + (np.uint64(2) * i + np.uint64(2)) * np.uint64(G))
    s = np.zeros(n, dtype=np.int64)
    for f in range(4):
        s += ((h0 >> np.uint64(16 * f)) & np.uint64(0xFFFF)).astype(np.int64)
        s += ((h1 >> np.uint64(16 * f)) & np.uint64(0xFFFF)).astype(np.int64)
    c = (2 * s - 8 * 65535).astype(np.float32)
    sc = np.frombuffer(struct.pack("<I", scale_bits(std)), dtype=np.float32)[0]
    return (c * sc).astype(np.float32)


def f32_to_bf16_bits(f: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest-even), returned as uint16 bit patterns."""
    u = f.astype(np.float32).view(np.uint32).astype(np.uint64)
    u = u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    return (u >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


# ---------------------------------------------------------------------------------------------
# build + load
# ---------------------------------------------------------------------------------------------
def build(verbose: bool = False) -> None:
    """Compile the host (gcc/OpenMP) and device (nvcc sm_100a) generators in-tree."""
    cmds = [
        ["gcc", "-O3", "-fopenmp", "-shared", "-fPIC", os.path.join(HERE, "synth_host.c"), "-o", HOST_LIB],
        ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-shared", "-Xcompiler", "-fPIC",
         os.path.join(HERE, "synth_dev.cu"), "-o", DEV_LIB],
    ]
    for c in cmds:
        if verbose:
            print(" ".join(c))
        subprocess.run(c, check=True)


_host = None
_dev = None


def host_lib():
    global _host
    if _host is None:
        if not os.path.exists(HOST_LIB):
            raise RuntimeError(f"{HOST_LIB} missing: run synth.build()")
        lib = ctypes.CDLL(HOST_LIB)
        u64, i64, u32, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_uint32, ctypes.c_void_p
        lib.synth_host_fill_f32.argtypes = [vp, i64, u64, u64, u64, u32]
        lib.synth_host_fill_bf16.argtypes = [vp, i64, u64, u64, u64, u32]
        lib.synth_host_hash.argtypes = [vp, i64, u64, u64]
        _host = lib
    return _host


def dev_lib():
    global _dev
    if _dev is None:
        if not os.path.exists(DEV_LIB):
            raise RuntimeError(f"{DEV_LIB} missing: run synth.build()")
        lib = ctypes.CDLL(DEV_LIB)
        u64, i64, u32, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_uint32, ctypes.c_void_p
        lib.synth_dev_fill_f32.argtypes = [vp, i64, u64, u64, u64, u32, vp]
        lib.synth_dev_fill_bf16.argtypes = [vp, i64, u64, u64, u64, u32, vp]
        lib.synth_dev_fill_f32.restype = ctypes.c_int
        lib.synth_dev_fill_bf16.restype = ctypes.c_int
        _dev = lib
    return _dev


# ---------------------------------------------------------------------------------------------
# host fills (numpy arrays; bf16 as uint16 bit patterns)
# ---------------------------------------------------------------------------------------------
def host_f32(n: int, seed: int, tid: int, std: float, index_base: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    host_lib().synth_host_fill_f32(out.ctypes.data, n, seed, tid, index_base, scale_bits(std))
    return out


def host_bf16(n: int, seed: int, tid: int, std: float, index_base: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.uint16)
    host_lib().synth_host_fill_bf16(out.ctypes.data, n, seed, tid, index_base, scale_bits(std))
    return out


def host_hash(n: int, seed: int, tid: int) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    host_lib().synth_host_hash(out.ctypes.data, n, seed, tid)
    return out


# ---------------------------------------------------------------------------------------------
# device fills (torch CUDA tensors)
# ---------------------------------------------------------------------------------------------
def _stream_handle(stream) -> int:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def dev_fill(t, seed: int, tid: int, std: float, index_base: int = 0, stream=None) -> None:
    """Fill a contiguous CUDA tensor (bf16 or fp32) with z(index_base + j)."""
    import torch
    assert t.is_cuda and t.is_contiguous()
    if t.dtype == torch.bfloat16:
        rc = dev_lib().synth_dev_fill_bf16(t.data_ptr(), t.numel(), seed, tid, index_base, scale_bits(std),
                                           _stream_handle(stream))
    elif t.dtype == torch.float32:
        rc = dev_lib().synth_dev_fill_f32(t.data_ptr(), t.numel(), seed, tid, index_base, scale_bits(std),
                                          _stream_handle(stream))
    else:
        raise TypeError(t.dtype)
    if rc != 0:
        raise RuntimeError(f"synth device fill failed: cudaError {rc}")


# ---------------------------------------------------------------------------------------------
# workload recipes
# ---------------------------------------------------------------------------------------------
@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    E: int
    k: int
    I: int
    Is: int
    route_scale: float = 3.0
    bias: str = "zero"            # "zero" | "zipf"
    spike_rows: int = 0           # rows of x scaled x spike_mult
    spike_mult: float = 50.0
    swiglu_limit: float = 0.0           # SwiGLU clamp of routed experts (0 = off)
    swiglu_limit_shared: float = 0.0    # SwiGLU clamp of the shared expert (0 = off)
    seed: int = 0
    x_std: float = 1.0
    w_std: float = 0.02
    description: str = field(default="", compare=False)


WORKLOADS = {
    "tiny": Workload("tiny", 64, 512, 32, 4, 128, 128,
                     description="T=64, H=512, E=32 top-4, I=Is=128, bias 0, seed 0"),
    "decode": Workload("decode", 64, 4096, 288, 8, 1280, 1280,
                       description="Step 3.5 Flash MoE layer, decode batch T=64, bias 0"),
    "prefill": Workload("prefill", 8192, 4096, 288, 8, 1280, 1280,
                        description="Step 3.5 Flash MoE layer, prefill T=8192, bias 0"),
    "skewed": Workload("skewed", 4096, 4096, 288, 8, 1280, 1280, bias="zipf",
                       description="T=4096, Zipf(1.2) expert popularity via router bias, 16 dead experts"),
    "mtp": Workload("mtp", 512, 4096, 288, 8, 1280, 1280, spike_rows=5,
                    description="MTP-3 verify batch 128x4=512 tokens, 1% of rows x50"),
    # the clamped variant of the deepest layers (model card swiglu_limits 7, swiglu_limits_shared
    # 16) on the MTP batch, whose x50 spike rows drive activations past the limits
    "mtp_clamp": Workload("mtp_clamp", 512, 4096, 288, 8, 1280, 1280, spike_rows=5, swiglu_limit=7.0,
                          swiglu_limit_shared=16.0,
                          description="MTP verify batch with the SwiGLU clamp (routed 7, shared 16)"),
    # profiling case: the decode kernel shape (~2 rows per expert) on 32 experts, ~1 GB of weights
    "decode_e32": Workload("decode_e32", 8, 4096, 32, 8, 1280, 1280,
                           description="decode-shaped small case for counter captures: T=8, 32 experts top-8"),
    # experiment case: the prefill GEMM shape with operands mostly L2-resident (8 experts x 2048 rows)
    "gemm_l2": Workload("gemm_l2", 8192, 4096, 8, 2, 1280, 1280,
                        description="8 experts top-2 over 8192 tokens: ~2048 rows per expert, weights reused from L2"),
    # profiling case: the prefill kernel shape (~225 rows per expert, token tile 256) on 32 experts
    "prefill_e32": Workload("prefill_e32", 900, 4096, 32, 8, 1280, 1280,
                            description="prefill-shaped small case for counter captures: T=900, 32 experts top-8"),
    # profiling case: the prefill kernel shape (~228 rows per expert, one 256-row tile each) with
    # several rounds of units per pair: 72 experts over 2048 tokens, ~2.6 GB on the device
    "prefill_e72": Workload("prefill_e72", 2048, 4096, 72, 8, 1280, 1280,
                            description="prefill-shaped steady-state case for counter captures: T=2048, 72 experts "
                                        "top-8"),
    # profiling case: the skewed batch's kernel shape (mean ~114 rows per expert, Zipf popularity
    # with 16 dead experts, 1-row to multi-tile groups) on 72 experts, ~2.3 GB of weights
    "skewed_e72": Workload("skewed_e72", 1024, 4096, 72, 8, 1280, 1280, bias="zipf",
                           description="skewed-shaped small case for counter captures: T=1024, 72 experts top-8, "
                                       "Zipf bias, 16 dead"),
}
ZIPF_DEAD = 16
ZIPF_FIXTURE = os.path.join(REPO, "tests", "golden", "zipf_bias.json")


def spike_rows(w: Workload) -> np.ndarray:
    """Rows of x scaled by spike_mult: the spike_rows rows with the smallest seeded hash."""
    if w.spike_rows == 0:
        return np.zeros(0, dtype=np.int64)
    h = host_hash(w.T, w.seed, TID_SPIKE_ROWS)
    return np.sort(np.argsort(h, kind="stable")[: w.spike_rows]).astype(np.int64)


def zipf_ranks(w: Workload) -> np.ndarray:
    """Popularity rank r_e in 1..E of each expert: experts ordered by their seeded hash."""
    h = host_hash(w.E, w.seed, TID_ZIPF_RANK)
    order = np.argsort(h, kind="stable")
    r = np.empty(w.E, dtype=np.int64)
    r[order] = np.arange(1, w.E + 1)
    return r


def zipf_bias(w: Workload, beta: float) -> np.ndarray:
    """bias_e = -beta * ln(r_e) for live ranks, -100 for the ZIPF_DEAD lowest ranks (never chosen)."""
    r = zipf_ranks(w)
    b = (-beta * np.log(r.astype(np.float64))).astype(np.float32)
    b[r > w.E - ZIPF_DEAD] = np.float32(-100.0)
    return b


def zipf_beta() -> float:
    with open(ZIPF_FIXTURE) as f:
        return float(json.load(f)["beta"])


def host_bias(w: Workload, beta: float | None = None) -> np.ndarray:
    if w.bias == "zero":
        return np.zeros(w.E, dtype=np.float32)
    if w.bias == "zipf":
        return zipf_bias(w, zipf_beta() if beta is None else beta)
    raise ValueError(w.bias)


def host_x_rows(w: Workload, rows: np.ndarray) -> np.ndarray:
    """bf16 bits of x for the given token rows, shape [len(rows), H]."""
    spikes = set(spike_rows(w).tolist())
    out = np.empty((len(rows), w.H), dtype=np.uint16)
    for i, t in enumerate(np.asarray(rows).tolist()):
        std = w.x_std * (w.spike_mult if t in spikes else 1.0)
        out[i] = host_bf16(w.H, w.seed, TID_X, std, index_base=t * w.H)
    return out


def host_x(w: Workload) -> np.ndarray:
    x = host_bf16(w.T * w.H, w.seed, TID_X, w.x_std).reshape(w.T, w.H)
    for t in spike_rows(w).tolist():
        x[t] = host_bf16(w.H, w.seed, TID_X, w.x_std * w.spike_mult, index_base=t * w.H)
    return x


def host_w_router(w: Workload) -> np.ndarray:
    return host_f32(w.E * w.H, w.seed, TID_WR, w.w_std).reshape(w.E, w.H)


def host_expert(w: Workload, e: int):
    """bf16 bits (W_g [I,H], W_u [I,H], W_d [H,I]) of routed expert e, or the shared expert when e == E."""
    if e == w.E:
        g = host_bf16(w.Is * w.H, w.seed, TID_WSG, w.w_std).reshape(w.Is, w.H)
        u = host_bf16(w.Is * w.H, w.seed, TID_WSU, w.w_std).reshape(w.Is, w.H)
        d = host_bf16(w.H * w.Is, w.seed, TID_WSD, w.w_std).reshape(w.H, w.Is)
        return g, u, d
    n = w.I * w.H
    g = host_bf16(n, w.seed, TID_WG, w.w_std, index_base=e * n).reshape(w.I, w.H)
    u = host_bf16(n, w.seed, TID_WU, w.w_std, index_base=e * n).reshape(w.I, w.H)
    d = host_bf16(n, w.seed, TID_WD, w.w_std, index_base=e * n).reshape(w.H, w.I)
    return g, u, d


# ---------------------------------------------------------------------------------------------
# device tensors for a workload (torch); weights in the library's logical layouts
# ---------------------------------------------------------------------------------------------
def dev_x(w: Workload, device="cuda"):
    import torch
    x = torch.empty(w.T, w.H, dtype=torch.bfloat16, device=device)
    dev_fill(x, w.seed, TID_X, w.x_std)
    for t in spike_rows(w).tolist():
        dev_fill(x[t], w.seed, TID_X, w.x_std * w.spike_mult, index_base=t * w.H)
    return x


def dev_router(w: Workload, device="cuda"):
    import torch
    wr = torch.empty(w.E, w.H, dtype=torch.float32, device=device)
    dev_fill(wr, w.seed, TID_WR, w.w_std)
    bias = torch.from_numpy(host_bias(w)).to(device)
    return wr, bias


def dev_experts(w: Workload, device="cuda"):
    """(W_g [E,I,H], W_u [E,I,H], W_d [E,H,I], Ws_g [Is,H], Ws_u [Is,H], Ws_d [H,Is]) as bf16 CUDA tensors."""
    import torch
    bf = torch.bfloat16
    wg = torch.empty(w.E, w.I, w.H, dtype=bf, device=device)
    wu = torch.empty(w.E, w.I, w.H, dtype=bf, device=device)
    wd = torch.empty(w.E, w.H, w.I, dtype=bf, device=device)
    sg = torch.empty(w.Is, w.H, dtype=bf, device=device)
    su = torch.empty(w.Is, w.H, dtype=bf, device=device)
    sd = torch.empty(w.H, w.Is, dtype=bf, device=device)
    for t, tid in ((wg, TID_WG), (wu, TID_WU), (wd, TID_WD), (sg, TID_WSG), (su, TID_WSU), (sd, TID_WSD)):
        dev_fill(t, w.seed, tid, w.w_std)
    return wg, wu, wd, sg, su, sd
