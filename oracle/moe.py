"""fp64 CPU oracle for one sparse MoE FFN layer of Step 3.5 Flash.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline / reference leg may import or call this module. The CUDA library
(``sparse_moe_layer_smoe_b200``) never imports it, and this module shares no code with it:
no kernels, headers, helpers, tables or pre/post-processing. Its only inputs are
plain numpy arrays (bf16 tensors as uint16 bit patterns, fp32 tensors as float32).

What the layer computes (sources, by page and section):

* Step-3.5-Flash model card (llm-atlas), raw config fields: ``hidden_size 4096``,
  ``moe_num_experts 288``, ``moe_top_k 8``, ``moe_intermediate_size 1280``,
  ``share_expert_dim 1280``, ``norm_expert_weight true``, ``moe_router_activation
  sigmoid``, ``moe_router_scaling_factor 3``, ``use_moe_router_bias true``,
  ``need_fp32_gate true``, ``torch_dtype bfloat16``.
* Step 3.5 Flash summary (hyper.ai), section "方法" (method): each MoE layer activates 8 of
  288 routed experts per token plus 1 shared expert.
* Step 3.5 Flash summary (paperlayer.ai), §2.2 "Sparse MoE Backbone with Hybrid Attention"
  (288 routed + 1 shared, top-8) and §4.1.2 "Expert Collapse Beyond Routing Collapse"
  (loss-free bias adjustment as the balancing device, so the bias steers selection).
* Same summary, §B "Detail Analysis of Localized Activation Blow-up": the expert is a
  SwiGLU with gate and up projections.

Readings where the pages are silent (each is also listed in the design notes):

1. the router bias is added to the sigmoid scores for *selection only*; combine weights
   come from the unbiased scores;
2. weights are the selected unbiased scores normalised to sum 1, then times 3;
3. the expert is SwiGLU: F(x) = W_d (SiLU(W_g x) * (W_u x)), SiLU(z) = z / (1 + e^-z);
4. the shared expert is added with weight 1 (no gate, no x3);
5. top-k order: biased score descending; equal biased scores -> larger raw logit first ->
   smaller expert index first;
6. a token is a near tie when its 8th and 9th biased scores differ by less than 1e-5; any
   selection within that band is correct there (``valid_selections``);
7. the layer output is the FFN output only (no residual, no norm);
8. SwiGLU clamp (model card fields ``swiglu_limits`` / ``swiglu_limits_shared``, garbled on the
   page; paperlayer.ai §4.1.3 and §B name activation clipping): with limit L > 0 the gate is
   clamped from above, min(g, L), and the up projection on both sides, clamp(u, -L, L), before
   SiLU(g) * u. L = 0 means no clamp. Routed and shared experts have their own limits.

Everything is computed in fp64 with no intermediate rounding. bf16 inputs and fp32 router
weights are exact in fp64.
"""
from __future__ import annotations

from dataclasses import dataclass
from itertools import combinations
from typing import Callable, Sequence

import numpy as np

NEAR_TIE_EPS = 1e-5


# ---------------------------------------------------------------------------------------------
# inputs
# ---------------------------------------------------------------------------------------------
def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact fp64 values."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def f32_to_f64(a: np.ndarray) -> np.ndarray:
    return np.asarray(a, dtype=np.float32).astype(np.float64)


# ---------------------------------------------------------------------------------------------
# router (model card: need_fp32_gate, moe_router_activation sigmoid, use_moe_router_bias,
#         moe_top_k, norm_expert_weight, moe_router_scaling_factor)
# ---------------------------------------------------------------------------------------------
def router_logits(x: np.ndarray, w_router: np.ndarray) -> np.ndarray:
    """L[t, e] = sum_h x[t, h] * W_r[e, h]  (fp64; x and W_r given as fp64)."""
    return x @ w_router.T


def sigmoid(z: np.ndarray) -> np.ndarray:
    """s = 1 / (1 + exp(-z))."""
    return 1.0 / (1.0 + np.exp(-z))


def select_topk(bhat: np.ndarray, logits: np.ndarray, k: int):
    """Per token, the k experts with the largest biased score, in descending order.

    Ties in the biased score are broken by the larger raw logit, then the smaller expert
    index (reading 5). Returns (idx [T, k] int32, gap [T]) where gap is the difference
    between the k-th and (k+1)-th biased scores (inf when E == k).
    """
    T, E = bhat.shape
    idx = np.empty((T, k), dtype=np.int32)
    gap = np.full(T, np.inf)
    experts = np.arange(E)
    for t in range(T):
        # np.lexsort sorts by the last key first
        order = np.lexsort((experts, -logits[t], -bhat[t]))
        idx[t] = order[:k]
        if E > k:
            gap[t] = bhat[t, order[k - 1]] - bhat[t, order[k]]
    return idx, gap


def normalise(s_sel: np.ndarray, scale: float) -> np.ndarray:
    """w_j = scale * (s_j / sum_j' s_j') over the selected (unbiased) scores: normalise, then scale
    (readings 1, 2)."""
    return scale * (s_sel / s_sel.sum(axis=-1, keepdims=True))


@dataclass
class Route:
    logits: np.ndarray   # [T, E]
    s: np.ndarray        # [T, E] sigmoid scores
    bhat: np.ndarray     # [T, E] biased scores used for selection
    idx: np.ndarray      # [T, k] int32, descending biased score
    w: np.ndarray        # [T, k] combine weights
    gap: np.ndarray      # [T] k-th minus (k+1)-th biased score

    @property
    def near_tie(self) -> np.ndarray:
        return self.gap < NEAR_TIE_EPS


def route(x: np.ndarray, w_router: np.ndarray, bias: np.ndarray, k: int, scale: float) -> Route:
    """Router: fp64 logits, sigmoid, bias for selection, top-k, renormalise x scale."""
    L = router_logits(x, w_router)
    s = sigmoid(L)
    bhat = s + bias[None, :]
    idx, gap = select_topk(bhat, L, k)
    s_sel = np.take_along_axis(s, idx.astype(np.int64), axis=1)
    return Route(L, s, bhat, idx, normalise(s_sel, scale), gap)


def valid_selections(bhat_row: np.ndarray, k: int, eps: float = NEAR_TIE_EPS):
    """All k-subsets S (as sorted tuples) with  min_{i in S} bhat_i >= max_{j not in S} bhat_j - eps.

    An expert whose biased score exceeds the (k+1)-th largest by more than eps is in every
    such S; one below the k-th largest by more than eps is in none. The rest are enumerated.
    """
    v = np.sort(bhat_row)[::-1]
    E = len(bhat_row)
    if E == k:
        return [tuple(range(E))]
    must = [e for e in range(E) if bhat_row[e] > v[k] + eps]
    cand = [e for e in range(E) if e not in must and bhat_row[e] >= v[k - 1] - eps]
    out = []
    for extra in combinations(cand, k - len(must)):
        S = set(must) | set(extra)
        lo = min(bhat_row[i] for i in S)
        hi = max((bhat_row[j] for j in range(E) if j not in S), default=-np.inf)
        if lo >= hi - eps:
            out.append(tuple(sorted(S)))
    return out


# ---------------------------------------------------------------------------------------------
# permutation (token -> expert dispatch)
# ---------------------------------------------------------------------------------------------
def permute(idx: np.ndarray, E: int):
    """Expert-major stable dispatch of the T*k (token, slot) entries.

    Entry p = t*k + j goes to row r; rows are ordered by expert, then token, then slot.
    Returns counts [E], offsets [E+1] (exclusive scan), perm_row [T*k] (entry -> row) and
    row_token [T*k] (row -> token).
    """
    T, k = idx.shape
    flat = idx.reshape(-1).astype(np.int64)
    order = np.argsort(flat, kind="stable")       # row r holds entry order[r]
    counts = np.bincount(flat, minlength=E).astype(np.int32)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    perm_row = np.empty(T * k, dtype=np.int32)
    perm_row[order] = np.arange(T * k, dtype=np.int32)
    row_token = (order // k).astype(np.int32)
    return counts, offsets, perm_row, row_token


# ---------------------------------------------------------------------------------------------
# experts (paperlayer §B: SwiGLU gate/up; model card: moe_intermediate_size, share_expert_dim)
# ---------------------------------------------------------------------------------------------
def silu(z: np.ndarray) -> np.ndarray:
    """SiLU(z) = z / (1 + exp(-z))."""
    return z / (1.0 + np.exp(-z))


def swiglu_hidden(X: np.ndarray, Wg: np.ndarray, Wu: np.ndarray, limit: float = 0.0) -> np.ndarray:
    """The SwiGLU hidden activation SiLU(W_g x) * (W_u x) for each row x of X; with limit L > 0
    the gate is clamped to (-inf, L] and the up projection to [-L, L] first (reading 8)."""
    G = X @ Wg.T
    U = X @ Wu.T
    if limit > 0.0:
        G = np.minimum(G, limit)
        U = np.clip(U, -limit, limit)
    return silu(G) * U


def swiglu_ffn(X: np.ndarray, Wg: np.ndarray, Wu: np.ndarray, Wd: np.ndarray, limit: float = 0.0) -> np.ndarray:
    """F(x) = W_d (SiLU(W_g x) * (W_u x)) for each row x of X (all fp64), clamped as in
    swiglu_hidden when limit > 0."""
    return swiglu_hidden(X, Wg, Wu, limit) @ Wd.T


ExpertFn = Callable[[int], Sequence[np.ndarray]]   # e -> (W_g, W_u, W_d) fp64; e == E is shared


def moe_sparse(x: np.ndarray, r: Route, expert: ExpertFn, E: int, limit: float = 0.0,
               limit_shared: float = 0.0) -> np.ndarray:
    """out[t] = F_shared(x_t) + sum_j w[t, j] F_{idx[t, j]}(x_t), computing only selected experts."""
    out = swiglu_ffn(x, *expert(E), limit=limit_shared)
    for e in np.unique(r.idx):
        rows, slots = np.nonzero(r.idx == e)
        out[rows] += r.w[rows, slots][:, None] * swiglu_ffn(x[rows], *expert(int(e)), limit=limit)
    return out


def moe_dense_masked(x: np.ndarray, r: Route, expert: ExpertFn, E: int, limit: float = 0.0,
                     limit_shared: float = 0.0) -> np.ndarray:
    """out[t] = F_shared(x_t) + sum_e m[t, e] w[t, e] F_e(x_t) over all E experts (0/1 mask m)."""
    T, k = r.idx.shape
    m = np.zeros((T, E))
    wfull = np.zeros((T, E))
    for j in range(k):
        m[np.arange(T), r.idx[:, j]] = 1.0
        wfull[np.arange(T), r.idx[:, j]] = r.w[:, j]
    out = swiglu_ffn(x, *expert(E), limit=limit_shared)
    for e in range(E):
        out += (m[:, e] * wfull[:, e])[:, None] * swiglu_ffn(x, *expert(e), limit=limit)
    return out


def moe_given_selection(x_t: np.ndarray, s_t: np.ndarray, sel: Sequence[int], expert: ExpertFn, E: int,
                        scale: float, limit: float = 0.0, limit_shared: float = 0.0) -> np.ndarray:
    """Output row of one token for a given selected set (used for near-tie tokens)."""
    sel = list(sel)
    w = normalise(s_t[sel], scale)
    out = swiglu_ffn(x_t[None, :], *expert(E), limit=limit_shared)[0]
    for wj, e in zip(w, sel):
        out = out + wj * swiglu_ffn(x_t[None, :], *expert(e), limit=limit)[0]
    return out


def combine(y: np.ndarray, perm_row: np.ndarray, w: np.ndarray, T: int, k: int) -> np.ndarray:
    """out[t] = y[T*k + t] + sum_j w[t, j] * y[perm_row[t*k + j]]  (y rows: routed, then shared)."""
    out = y[T * k: T * k + T].copy()
    pr = perm_row.reshape(T, k)
    for j in range(k):
        out += w[:, j:j + 1] * y[pr[:, j]]
    return out
