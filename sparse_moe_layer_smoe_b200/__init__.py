"""Python binding for libstepmoe: the C-ABI of include/stepmoe.h, same names, argument marshalling only.

Every step of the layer runs in the library's CUDA kernels; this module only turns torch
tensors (or raw integers) into pointers and checks the returned status. PyTorch supplies
device memory and streams. If ``libstepmoe.so`` is missing the binding raises: there is no
fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os
import re
from dataclasses import dataclass

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libstepmoe.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "stepmoe.h")

STATUS = {0: "SMOE_OK", 1: "SMOE_ERR_INVALID_ARG", 2: "SMOE_ERR_UNSUPPORTED", 3: "SMOE_ERR_WORKSPACE",
          4: "SMOE_ERR_CUDA", 5: "SMOE_ERR_DEVICE", 6: "SMOE_ERR_TIMEOUT"}
SMOE_OK, SMOE_ERR_INVALID_ARG, SMOE_ERR_UNSUPPORTED, SMOE_ERR_WORKSPACE = 0, 1, 2, 3
SMOE_ERR_CUDA, SMOE_ERR_DEVICE, SMOE_ERR_TIMEOUT = 4, 5, 6
SMOE_NOALLOC_SCRATCH_BYTES = 16 << 20   # include/stepmoe.h: the allocation-free router's static scratch


class SmoeConfig(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("n_experts", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("inter", ctypes.c_int32), ("shared_inter", ctypes.c_int32), ("route_scale", ctypes.c_float),
                ("swiglu_limit", ctypes.c_float), ("swiglu_limit_shared", ctypes.c_float)]


class SmoeError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {STATUS.get(status, status)}")
        self.status = status


def config(hidden=4096, n_experts=288, top_k=8, inter=1280, shared_inter=1280, route_scale=3.0,
           swiglu_limit=0.0, swiglu_limit_shared=0.0) -> SmoeConfig:
    return SmoeConfig(hidden, n_experts, top_k, inter, shared_inter, route_scale, swiglu_limit, swiglu_limit_shared)


class SmoeKernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int32), ("total_ms", ctypes.c_float)]


class SmoeDiag(ctypes.Structure):
    """smoe_diag_t: device pointers of the monitoring outputs (see include/stepmoe.h)."""
    _fields_ = [("expert_count", ctypes.c_void_p), ("expert_norm_mean", ctypes.c_void_p),
                ("expert_norm_max", ctypes.c_void_p), ("token_confidence", ctypes.c_void_p),
                ("summary", ctypes.c_void_p)]


# indices into smoe_diag_t.summary
(SMOE_DIAG_ACTIVE_EXPERTS, SMOE_DIAG_NORM_MEDIAN, SMOE_DIAG_NORM_MAX_TO_MEDIAN, SMOE_DIAG_NORM_MIN_TO_MEDIAN,
 SMOE_DIAG_CONF_MEAN, SMOE_DIAG_CONF_MIN, SMOE_DIAG_LOAD_MAX_TO_MEAN, SMOE_DIAG_NORM_PEAK, SMOE_DIAG_SUMMARY) = range(9)
DIAG_FIELDS = ("expert_count", "expert_norm_mean", "expert_norm_max", "token_confidence", "summary")


_vp, _i64, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
_cfgp = ctypes.POINTER(SmoeConfig)
_SIGS = {
    "smoe_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "smoe_check_config": ([_cfgp], ctypes.c_int),
    "smoe_scratch_bytes": ([_cfgp, _i64, ctypes.POINTER(_sz)], ctypes.c_int),
    "smoe_workspace_bytes": ([_cfgp, _i64, ctypes.POINTER(_sz)], ctypes.c_int),
    "smoe_packed_weight_bytes": ([_cfgp, ctypes.POINTER(_sz)], ctypes.c_int),
    "smoe_pack_weights": ([_cfgp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp], ctypes.c_int),
    "smoe_route": ([_cfgp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp], ctypes.c_int),
    "smoe_permute": ([_cfgp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp], ctypes.c_int),
    "smoe_expert_ffn": ([_cfgp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _sz, _vp], ctypes.c_int),
    "smoe_combine": ([_cfgp, _vp, _vp, _vp, _i64, _vp, _vp, _sz, _vp], ctypes.c_int),
    "smoe_forward": ([_cfgp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _sz, _vp], ctypes.c_int),
    "smoe_forward_diag": ([_cfgp, _vp, _i64, _vp, _vp, _vp, _vp, ctypes.POINTER(SmoeDiag), _vp, _sz, _vp],
                          ctypes.c_int),
    "smoe_get_device_error": ([_vp, ctypes.POINTER(ctypes.c_int32), _vp], ctypes.c_int),
    "smoe_clear_device_error": ([_vp, _vp], ctypes.c_int),
    "smoe_last_launch_count": ([], ctypes.c_int32),
    "smoe_timing_begin": ([ctypes.c_int32], ctypes.c_int),
    "smoe_timing_end": ([ctypes.POINTER(SmoeKernelTime), ctypes.c_int32, ctypes.POINTER(ctypes.c_int32)],
                        ctypes.c_int),
    "smoe_route_noalloc": ([_cfgp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp], ctypes.c_int),
    "smoe_packed_weight_bytes_fp8": ([_cfgp, ctypes.POINTER(_sz)], ctypes.c_int),
    "smoe_pack_weights_fp8": ([_cfgp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp], ctypes.c_int),
    "smoe_workspace_bytes_fp8": ([_cfgp, _i64, ctypes.POINTER(_sz)], ctypes.c_int),
    "smoe_forward_fp8": ([_cfgp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _sz, _vp], ctypes.c_int),
    "smoe_selftest_wait_timeout": ([ctypes.c_uint64, _vp, _vp, _vp], ctypes.c_int),
    "smoe_selftest_swiglu": ([_vp, _vp, _i64, _vp, _vp], ctypes.c_int),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load libstepmoe.so (built in-tree). Raises if it is missing: the layer has no other path."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with sparse_moe_layer_smoe_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of the functions include/stepmoe.h declares."""
    with open(HEADER) as f:
        text = f.read()
    return re.findall(r"^SMOE_API\s+[\w\s\*]*?\b(smoe_\w+)\s*\(", text, flags=re.M)


def _p(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _s(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream or None
    if isinstance(stream, int):
        return stream or None
    return stream.cuda_stream or None


def _check(name: str, status: int) -> None:
    if status != SMOE_OK:
        raise SmoeError(name, status)


def _bytes(fn, cfg, *args) -> int:
    out = _sz(0)
    _check(fn.__name__, fn(ctypes.byref(cfg), *args, ctypes.byref(out)))
    return out.value


# ------------------------------------------------------------------------------ same-name wrappers
def smoe_status_string(status: int) -> str:
    return lib().smoe_status_string(status).decode()


def smoe_check_config(cfg: SmoeConfig) -> int:
    return lib().smoe_check_config(ctypes.byref(cfg))


def smoe_scratch_bytes(cfg: SmoeConfig, T: int) -> int:
    return _bytes(lib().smoe_scratch_bytes, cfg, T)


def smoe_workspace_bytes(cfg: SmoeConfig, T: int) -> int:
    return _bytes(lib().smoe_workspace_bytes, cfg, T)


def smoe_packed_weight_bytes(cfg: SmoeConfig) -> int:
    return _bytes(lib().smoe_packed_weight_bytes, cfg)


def smoe_pack_weights(cfg, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, packed, stream=None) -> None:
    _check("smoe_pack_weights", lib().smoe_pack_weights(ctypes.byref(cfg), _p(w_gate), _p(w_up), _p(w_down),
                                                         _p(ws_gate), _p(ws_up), _p(ws_down), _p(packed), _s(stream)))


def smoe_route(cfg, x, T, w_router, bias, topk_idx, topk_w, logits=None, ws=None, ws_bytes=None, stream=None):
    _check("smoe_route", lib().smoe_route(ctypes.byref(cfg), _p(x), T, _p(w_router), _p(bias), _p(topk_idx),
                                          _p(topk_w), _p(logits), _p(ws), _ws_bytes(ws, ws_bytes), _s(stream)))


def smoe_route_noalloc(cfg, x, T, w_router, bias, topk_idx, topk_w, logits=None, stream=None):
    """smoe_route without a workspace (library-owned static scratch; see include/stepmoe.h)."""
    _check("smoe_route_noalloc", lib().smoe_route_noalloc(ctypes.byref(cfg), _p(x), T, _p(w_router), _p(bias),
                                                          _p(topk_idx), _p(topk_w), _p(logits), _s(stream)))


def smoe_permute(cfg, topk_idx, T, x, counts, offsets, perm_row, row_token, x_perm, ws=None, ws_bytes=None,
                 stream=None):
    _check("smoe_permute", lib().smoe_permute(ctypes.byref(cfg), _p(topk_idx), T, _p(x), _p(counts), _p(offsets),
                                              _p(perm_row), _p(row_token), _p(x_perm), _p(ws),
                                              _ws_bytes(ws, ws_bytes), _s(stream)))


def smoe_expert_ffn(cfg, x, x_perm, row_token, offsets, T, packed, y, ws=None, ws_bytes=None, stream=None):
    _check("smoe_expert_ffn", lib().smoe_expert_ffn(ctypes.byref(cfg), _p(x), _p(x_perm), _p(row_token),
                                                    _p(offsets), T, _p(packed), _p(y), _p(ws),
                                                    _ws_bytes(ws, ws_bytes), _s(stream)))


def smoe_combine(cfg, y, perm_row, topk_w, T, out, ws=None, ws_bytes=None, stream=None):
    _check("smoe_combine", lib().smoe_combine(ctypes.byref(cfg), _p(y), _p(perm_row), _p(topk_w), T, _p(out),
                                              _p(ws), _ws_bytes(ws, ws_bytes), _s(stream)))


def smoe_forward(cfg, x, T, w_router, bias, packed, out, ws=None, ws_bytes=None, stream=None):
    _check("smoe_forward", lib().smoe_forward(ctypes.byref(cfg), _p(x), T, _p(w_router), _p(bias), _p(packed),
                                              _p(out), _p(ws), _ws_bytes(ws, ws_bytes), _s(stream)))


def smoe_forward_diag(cfg, x, T, w_router, bias, packed, out, diag, ws=None, ws_bytes=None, stream=None):
    """diag: a mapping with the smoe_diag_t fields (device tensors), e.g. from diag_buffers()."""
    d = SmoeDiag(*[_p(diag[f]) for f in DIAG_FIELDS])
    _check("smoe_forward_diag", lib().smoe_forward_diag(ctypes.byref(cfg), _p(x), T, _p(w_router), _p(bias),
                                                        _p(packed), _p(out), ctypes.byref(d), _p(ws),
                                                        _ws_bytes(ws, ws_bytes), _s(stream)))


def smoe_packed_weight_bytes_fp8(cfg: SmoeConfig) -> int:
    return _bytes(lib().smoe_packed_weight_bytes_fp8, cfg)


def smoe_workspace_bytes_fp8(cfg: SmoeConfig, T: int) -> int:
    return _bytes(lib().smoe_workspace_bytes_fp8, cfg, T)


def smoe_pack_weights_fp8(cfg, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, packed, stream=None) -> None:
    _check("smoe_pack_weights_fp8", lib().smoe_pack_weights_fp8(ctypes.byref(cfg), _p(w_gate), _p(w_up), _p(w_down),
                                                                 _p(ws_gate), _p(ws_up), _p(ws_down), _p(packed),
                                                                 _s(stream)))


def smoe_forward_fp8(cfg, x, T, w_router, bias, packed_fp8, out, ws=None, ws_bytes=None, stream=None):
    _check("smoe_forward_fp8", lib().smoe_forward_fp8(ctypes.byref(cfg), _p(x), T, _p(w_router), _p(bias),
                                                      _p(packed_fp8), _p(out), _p(ws), _ws_bytes(ws, ws_bytes),
                                                      _s(stream)))


def smoe_selftest_swiglu(g, u, n, out, stream=None) -> None:
    """The expert epilogue's SiLU(g) * u (see include/stepmoe.h)."""
    _check("smoe_selftest_swiglu", lib().smoe_selftest_swiglu(_p(g), _p(u), int(n), _p(out), _s(stream)))


def smoe_selftest_wait_timeout(limit_ns, elapsed_ns=None, ws=None, stream=None) -> None:
    _check("smoe_selftest_wait_timeout", lib().smoe_selftest_wait_timeout(int(limit_ns), _p(elapsed_ns), _p(ws),
                                                                          _s(stream)))


def smoe_get_device_error(ws, stream=None) -> int:
    code = ctypes.c_int32(0)
    _check("smoe_get_device_error", lib().smoe_get_device_error(_p(ws), ctypes.byref(code), _s(stream)))
    return code.value


def smoe_clear_device_error(ws, stream=None) -> None:
    _check("smoe_clear_device_error", lib().smoe_clear_device_error(_p(ws), _s(stream)))


def smoe_last_launch_count() -> int:
    return int(lib().smoe_last_launch_count())


def smoe_timing_begin(max_launches: int) -> None:
    _check("smoe_timing_begin", lib().smoe_timing_begin(max_launches))


def smoe_timing_end() -> dict:
    """{kernel name: (launches, total_ms)} for the launches recorded since smoe_timing_begin."""
    buf = (SmoeKernelTime * 16)()
    n = ctypes.c_int32(0)
    _check("smoe_timing_end", lib().smoe_timing_end(buf, 16, ctypes.byref(n)))
    return {buf[i].name.decode(): (int(buf[i].launches), float(buf[i].total_ms)) for i in range(n.value)}


def _ws_bytes(ws, ws_bytes) -> int:
    if ws_bytes is not None:
        return int(ws_bytes)
    if ws is None or isinstance(ws, int):
        return 0
    return ws.numel() * ws.element_size()


# ------------------------------------------------------------------------------ conveniences (torch memory)
def workspace(cfg: SmoeConfig, T: int, forward: bool = True, device="cuda", fp8: bool = False):
    """A zeroed uint8 CUDA tensor large enough for smoe_forward (smoe_forward_fp8 with fp8=True,
    or the per-call entry points with forward=False)."""
    import torch
    if fp8:
        n = smoe_workspace_bytes_fp8(cfg, T)
    else:
        n = smoe_workspace_bytes(cfg, T) if forward else smoe_scratch_bytes(cfg, T)
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=device)


def diag_buffers(cfg: SmoeConfig, T: int, device="cuda") -> dict:
    """Device arrays for smoe_forward_diag's outputs."""
    import torch
    E = cfg.n_experts
    return {"expert_count": torch.empty(E, dtype=torch.int32, device=device),
            "expert_norm_mean": torch.empty(E, dtype=torch.float32, device=device),
            "expert_norm_max": torch.empty(E, dtype=torch.float32, device=device),
            "token_confidence": torch.empty(max(T, 1), dtype=torch.float32, device=device),
            "summary": torch.empty(SMOE_DIAG_SUMMARY, dtype=torch.float32, device=device)}


def pack_weights(cfg, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, stream=None):
    import torch
    packed = torch.empty(smoe_packed_weight_bytes(cfg), dtype=torch.uint8, device=w_gate.device)
    smoe_pack_weights(cfg, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, packed, stream)
    return packed


def pack_weights_fp8(cfg, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, stream=None):
    import torch
    packed = torch.empty(smoe_packed_weight_bytes_fp8(cfg), dtype=torch.uint8, device=w_gate.device)
    smoe_pack_weights_fp8(cfg, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, packed, stream)
    return packed


@dataclass
class MoELayer:
    """Parameters of one layer on the device: fp32 router weights and bias, packed bf16 experts."""
    cfg: SmoeConfig
    w_router: object
    bias: object
    packed: object

    def forward(self, x, out=None, ws=None, stream=None):
        import torch
        T = x.shape[0]
        if out is None:
            out = torch.empty(T, self.cfg.hidden, dtype=torch.bfloat16, device=x.device)
        if ws is None:
            ws = workspace(self.cfg, T, device=x.device)
        smoe_forward(self.cfg, x, T, self.w_router, self.bias, self.packed, out, ws, stream=stream)
        return out
