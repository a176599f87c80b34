"""Python face of the C++ fp64 oracle (``smoe_oracle.cpp``) — TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and reference legs
may import this module. It marshals numpy arrays into the C++ library and back; every step of
the layer (router, sigmoid, top-k, weights, dispatch, SwiGLU experts, combine) is computed in the
C++ code. The library is compiled with g++ (plain C++17, ``-ffp-contract=off``, no BLAS) into
``oracle/libsmoe_oracle.so`` on first use when it is missing or older than its source.

The functions have the names and signatures of the numpy restatement in ``oracle/moe.py``, so a
test can run against either; ``oracle`` (the package) exports these C++ ones.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Sequence

import numpy as np

from .moe import NEAR_TIE_EPS, ExpertFn, Route

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "smoe_oracle.cpp")
LIB = os.path.join(HERE, "libsmoe_oracle.so")
CXX_FLAGS = ["-O2", "-std=c++17", "-ffp-contract=off", "-fPIC", "-shared", "-pthread", "-Wall"]

_lib = None
_lock = threading.Lock()

_d = ctypes.POINTER(ctypes.c_double)
_i32 = ctypes.POINTER(ctypes.c_int32)
_pd = ctypes.POINTER(_d)
EXPERT_FN = ctypes.CFUNCTYPE(ctypes.c_int, ctypes.c_void_p, ctypes.c_int32, _pd, _pd, _pd)


def build(src: str = SRC, out: str = LIB, verbose: bool = False) -> str:
    """Compile the C++ oracle into a shared library."""
    cmd = ["g++", *CXX_FLAGS, src, "-o", out]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    return out


def load(path: str):
    """Load a compiled oracle library and declare its entry points."""
    lib = ctypes.CDLL(path)
    i64, i32, f64, vp = ctypes.c_int64, ctypes.c_int32, ctypes.c_double, ctypes.c_void_p
    sig = {
        "so_set_threads": (None, [i32]),
        "so_threads": (i32, []),
        "so_bf16_to_f64": (None, [vp, i64, vp]),
        "so_f32_to_f64": (None, [vp, i64, vp]),
        "so_sigmoid": (None, [vp, i64, vp]),
        "so_silu": (None, [vp, i64, vp]),
        "so_router_logits": (ctypes.c_int, [vp, i64, i64, vp, i64, vp]),
        "so_select_topk": (ctypes.c_int, [vp, vp, i64, i32, i32, vp, vp]),
        "so_normalise": (ctypes.c_int, [vp, i64, i32, f64, vp]),
        "so_route": (ctypes.c_int, [vp, i64, i64, vp, i32, vp, i32, f64, vp, vp, vp, vp, vp, vp]),
        "so_valid_selections": (i64, [vp, i32, i32, f64, vp, i64]),
        "so_permute": (ctypes.c_int, [vp, i64, i32, i32, vp, vp, vp, vp]),
        "so_swiglu_hidden": (ctypes.c_int, [vp, i64, i64, vp, vp, i64, f64, vp]),
        "so_swiglu_ffn": (ctypes.c_int, [vp, i64, i64, vp, vp, vp, i64, f64, vp]),
        "so_moe": (ctypes.c_int, [i32, vp, i64, i64, i32, i32, i64, vp, vp, EXPERT_FN, vp, f64, f64, vp]),
        "so_moe_given_selection": (ctypes.c_int, [vp, vp, vp, i32, i64, i32, i64, f64, EXPERT_FN, vp, f64, f64,
                                                  vp]),
        "so_combine": (ctypes.c_int, [vp, vp, vp, i64, i32, i64, vp]),
        "so_forward_timed": (ctypes.c_int, [vp, i64, i64, vp, i32, vp, i32, f64, i64, EXPERT_FN, vp, f64, f64, i32,
                                            vp, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def lib():
    """The oracle library, compiled first if it is missing or older than its source."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
                build()
            _lib = load(LIB)
        return _lib


def set_threads(n: int) -> None:
    """Worker threads of the C++ oracle (0: all hardware threads)."""
    lib().so_set_threads(int(n))


def threads() -> int:
    return int(lib().so_threads())


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _i32a(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.int32)


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError(f"oracle {what} failed with code {rc}")


# ------------------------------------------------------------------------------------------ inputs
def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact fp64 values."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(b.shape, dtype=np.float64)
    lib().so_bf16_to_f64(_p(b), b.size, _p(out))
    return out


def f32_to_f64(a: np.ndarray) -> np.ndarray:
    f = np.ascontiguousarray(a, dtype=np.float32)
    out = np.empty(f.shape, dtype=np.float64)
    lib().so_f32_to_f64(_p(f), f.size, _p(out))
    return out


# ------------------------------------------------------------------------------------------ router
def sigmoid(z) -> np.ndarray:
    z = _f64(z)
    out = np.empty_like(z)
    lib().so_sigmoid(_p(z), z.size, _p(out))
    return out


def silu(z) -> np.ndarray:
    z = _f64(z)
    out = np.empty_like(z)
    lib().so_silu(_p(z), z.size, _p(out))
    return out


def router_logits(x: np.ndarray, w_router: np.ndarray) -> np.ndarray:
    x, wr = _f64(x), _f64(w_router)
    T, H = x.shape
    L = np.empty((T, wr.shape[0]))
    _check(lib().so_router_logits(_p(x), T, H, _p(wr), wr.shape[0], _p(L)), "router_logits")
    return L


def select_topk(bhat: np.ndarray, logits: np.ndarray, k: int):
    bhat, logits = _f64(bhat), _f64(logits)
    T, E = bhat.shape
    idx = np.empty((T, k), dtype=np.int32)
    gap = np.empty(T)
    _check(lib().so_select_topk(_p(bhat), _p(logits), T, E, k, _p(idx), _p(gap)), "select_topk")
    return idx, gap


def normalise(s_sel: np.ndarray, scale: float) -> np.ndarray:
    """w_j = scale * (s_j / sum_j' s_j') over the last axis (the selected unbiased scores)."""
    s_sel = _f64(s_sel)
    k = s_sel.shape[-1]
    n = s_sel.size // k
    out = np.empty_like(s_sel)
    _check(lib().so_normalise(_p(s_sel), n, k, float(scale), _p(out)), "normalise")
    return out


def route(x: np.ndarray, w_router: np.ndarray, bias: np.ndarray, k: int, scale: float) -> Route:
    """Router: fp64 logits, sigmoid, bias for selection, top-k, renormalise x scale."""
    x, wr, bias = _f64(x), _f64(w_router), _f64(bias)
    T, H = x.shape
    E = wr.shape[0]
    L, s, bhat = np.empty((T, E)), np.empty((T, E)), np.empty((T, E))
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k))
    gap = np.empty(T)
    _check(lib().so_route(_p(x), T, H, _p(wr), E, _p(bias), k, float(scale), _p(L), _p(s), _p(bhat), _p(idx), _p(w),
                          _p(gap)), "route")
    return Route(L, s, bhat, idx, w, gap)


def valid_selections(bhat_row: np.ndarray, k: int, eps: float = NEAR_TIE_EPS):
    """All k-subsets S (sorted tuples) with min_{i in S} bhat_i >= max_{j not in S} bhat_j - eps."""
    row = _f64(bhat_row)
    E = row.size
    cap = 64
    while True:
        sets = np.empty((cap, k), dtype=np.int32)
        n = int(lib().so_valid_selections(_p(row), E, k, float(eps), _p(sets), cap))
        if n < 0:
            raise ValueError("oracle valid_selections: bad arguments")
        if n <= cap:
            return [tuple(int(v) for v in sets[i]) for i in range(n)]
        cap = n


# ------------------------------------------------------------------------------------------ dispatch
def permute(idx: np.ndarray, E: int):
    """Expert-major stable dispatch: counts [E], offsets [E+1], perm_row [T*k], row_token [T*k]."""
    idx = _i32a(idx)
    T, k = idx.shape
    counts = np.empty(E, dtype=np.int32)
    offsets = np.empty(E + 1, dtype=np.int32)
    perm_row = np.empty(T * k, dtype=np.int32)
    row_token = np.empty(T * k, dtype=np.int32)
    _check(lib().so_permute(_p(idx), T, k, E, _p(counts), _p(offsets), _p(perm_row), _p(row_token)), "permute")
    return counts, offsets, perm_row, row_token


# ------------------------------------------------------------------------------------------ experts
def swiglu_hidden(X: np.ndarray, Wg: np.ndarray, Wu: np.ndarray, limit: float = 0.0) -> np.ndarray:
    X, Wg, Wu = _f64(X), _f64(Wg), _f64(Wu)
    n, H = X.shape
    I = Wg.shape[0]
    hid = np.empty((n, I))
    _check(lib().so_swiglu_hidden(_p(X), n, H, _p(Wg), _p(Wu), I, float(limit), _p(hid)), "swiglu_hidden")
    return hid


def swiglu_ffn(X: np.ndarray, Wg: np.ndarray, Wu: np.ndarray, Wd: np.ndarray, limit: float = 0.0) -> np.ndarray:
    X, Wg, Wu, Wd = _f64(X), _f64(Wg), _f64(Wu), _f64(Wd)
    n, H = X.shape
    I = Wg.shape[0]
    Y = np.empty((n, H))
    _check(lib().so_swiglu_ffn(_p(X), n, H, _p(Wg), _p(Wu), _p(Wd), I, float(limit), _p(Y)), "swiglu_ffn")
    return Y


class _Fetcher:
    """The C++ layer's expert callback: fp64 weights of expert e from a Python ExpertFn, kept alive
    until the next request."""

    def __init__(self, expert: ExpertFn):
        self.expert = expert
        self.held = None
        self.error = None
        self.I = None
        self.fn = EXPERT_FN(self._fetch)

    def _fetch(self, _ctx, e, pg, pu, pd):
        try:
            wg, wu, wd = (_f64(a) for a in self.expert(int(e)))
            if self.I is not None and wg.shape[0] != self.I:
                raise ValueError(f"expert {e}: inter {wg.shape[0]} != {self.I}")
            self.held = (wg, wu, wd)
            pg[0] = wg.ctypes.data_as(_d)
            pu[0] = wu.ctypes.data_as(_d)
            pd[0] = wd.ctypes.data_as(_d)
            return 0
        except Exception as exc:   # reported after the C++ call returns
            self.error = exc
            return 1


def _moe(dense: bool, x, r: Route, expert: ExpertFn, E: int, limit: float, limit_shared: float) -> np.ndarray:
    x = _f64(x)
    T, H = x.shape
    idx, w = _i32a(r.idx), _f64(r.w)
    k = idx.shape[1]
    f = _Fetcher(expert)
    I = _f64(expert(E)[0]).shape[0]
    f.I = I
    out = np.empty((T, H))
    rc = lib().so_moe(int(dense), _p(x), T, H, E, k, I, _p(idx), _p(w), f.fn, None, float(limit),
                      float(limit_shared), _p(out))
    if f.error is not None:
        raise f.error
    _check(rc, "moe")
    return out


def moe_sparse(x: np.ndarray, r: Route, expert: ExpertFn, E: int, limit: float = 0.0,
               limit_shared: float = 0.0) -> np.ndarray:
    """out[t] = F_shared(x_t) + sum_j w[t, j] F_{idx[t, j]}(x_t), computing only selected experts."""
    return _moe(False, x, r, expert, E, limit, limit_shared)


def moe_dense_masked(x: np.ndarray, r: Route, expert: ExpertFn, E: int, limit: float = 0.0,
                     limit_shared: float = 0.0) -> np.ndarray:
    """out[t] = F_shared(x_t) + sum_e m[t, e] w[t, e] F_e(x_t) over all E experts (0/1 mask m)."""
    return _moe(True, x, r, expert, E, limit, limit_shared)


def moe_given_selection(x_t: np.ndarray, s_t: np.ndarray, sel: Sequence[int], expert: ExpertFn, E: int,
                        scale: float, limit: float = 0.0, limit_shared: float = 0.0) -> np.ndarray:
    """Output row of one token for a given selected set (used for near-tie tokens)."""
    x_t, s_t = _f64(x_t).reshape(-1), _f64(s_t).reshape(-1)
    sel = _i32a(list(sel))
    H = x_t.size
    f = _Fetcher(expert)
    I = _f64(expert(E)[0]).shape[0]
    f.I = I
    out = np.empty(H)
    rc = lib().so_moe_given_selection(_p(x_t), _p(s_t), _p(sel), sel.size, H, E, I, float(scale), f.fn, None,
                                      float(limit), float(limit_shared), _p(out))
    if f.error is not None:
        raise f.error
    _check(rc, "moe_given_selection")
    return out


def combine(y: np.ndarray, perm_row: np.ndarray, w: np.ndarray, T: int, k: int) -> np.ndarray:
    """out[t] = y[T*k + t] + sum_j w[t, j] * y[perm_row[t*k + j]]  (y rows: routed, then shared)."""
    y, pr, w = _f64(y), _i32a(perm_row), _f64(w)
    H = y.shape[1]
    out = np.empty((T, H))
    _check(lib().so_combine(_p(y), _p(pr), _p(w), T, k, H, _p(out)), "combine")
    return out


def forward_timed(x: np.ndarray, w_router: np.ndarray, bias: np.ndarray, k: int, scale: float,
                  expert: ExpertFn, E: int, repeats: int, limit: float = 0.0, limit_shared: float = 0.0):
    """``repeats`` passes of route + the sparse layer, timed inside the C++ code with
    std::chrono::steady_clock. Returns (output, seconds)."""
    x, wr, bias = _f64(x), _f64(w_router), _f64(bias)
    T, H = x.shape
    f = _Fetcher(expert)
    I = _f64(expert(E)[0]).shape[0]
    f.I = I
    out = np.empty((T, H))
    sec = np.zeros(1)
    rc = lib().so_forward_timed(_p(x), T, H, _p(wr), E, _p(bias), k, float(scale), I, f.fn, None, float(limit),
                                float(limit_shared), int(repeats), _p(out), _p(sec))
    if f.error is not None:
        raise f.error
    _check(rc, "forward_timed")
    return out, float(sec[0])
