"""fp64 oracle of the layer's monitoring outputs (the diagnostics side outputs).

TEST INFRASTRUCTURE, like the rest of ``oracle/``: only ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU leg may import it; the CUDA library shares no code with it.

Sources (Step 3.5 Flash summary, paperlayer.ai):

* §4.1.2 "Expert Collapse Beyond Routing Collapse": monitor per-expert activation norms; a
  falling minimum-to-median ratio of them warns of expert death;
* §4.1.3 "Localized Activation Blow-up in MoE Layers": the maximum-to-median activation-norm
  ratio exposes blow-up in a few experts while the median norm stays flat;
* §5.2.1 "MIS-Filtered Policy Optimization": routing confidence as a proxy for MoE stability.

Readings (the pages give no formulas):

1. the activation norm of expert e for token t is ||F_e(x_t)||_2, the L2 norm of the routed
   expert's output row, before its routing weight; per expert, the mean and the max over the
   tokens routed to it (0 for an expert without tokens);
2. the ratios are taken over the experts that received tokens, against the median of their
   mean norms (for an even count, the mean of the two middle values); 0 when the median is 0;
3. the routing confidence of token t is the mean of its k selected unbiased sigmoid scores;
4. the load ratio is the largest per-expert count over the mean count T k / E.

Every value here is fp64 from the oracle's own expert outputs (no rounding). The GPU takes
the norm of its bf16 output rows, which the tests allow for.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .moe import ExpertFn, Route, swiglu_ffn

SUMMARY_FIELDS = ("active_experts", "norm_median", "norm_max_to_median", "norm_min_to_median", "conf_mean",
                  "conf_min", "load_max_to_mean", "norm_peak")


@dataclass
class Diagnostics:
    expert_count: np.ndarray      # [E] int
    expert_norm_mean: np.ndarray  # [E]
    expert_norm_max: np.ndarray   # [E]
    token_confidence: np.ndarray  # [T]
    summary: np.ndarray           # [8], in SUMMARY_FIELDS order
    row_norm: np.ndarray          # [T, k]: ||F_{idx[t, j]}(x_t)||_2


def expert_output_norms(x: np.ndarray, r: Route, expert: ExpertFn, limit: float = 0.0) -> np.ndarray:
    """[T, k]: the L2 norm of each selected expert's output row for its token (reading 1)."""
    T, k = r.idx.shape
    norms = np.zeros((T, k))
    for e in np.unique(r.idx):
        rows, slots = np.nonzero(r.idx == e)
        y = swiglu_ffn(x[rows], *expert(int(e)), limit=limit)
        norms[rows, slots] = np.sqrt(np.sum(y * y, axis=1))
    return norms


def summarise(count: np.ndarray, norm_mean: np.ndarray, norm_max: np.ndarray, conf: np.ndarray, T: int,
              k: int) -> np.ndarray:
    """The layer summary from per-expert statistics and token confidences (readings 2-4)."""
    E = count.shape[0]
    active = count > 0
    n = int(active.sum())
    med = float(np.median(norm_mean[active])) if n > 0 else 0.0
    hi = float(norm_mean[active].max()) if n > 0 else 0.0
    lo = float(norm_mean[active].min()) if n > 0 else 0.0
    return np.array([n, med, hi / med if med > 0 else 0.0, lo / med if med > 0 else 0.0, float(conf.mean()),
                     float(conf.min()), float(count.max()) / (T * k / E), float(norm_max.max())])


def diagnostics(x: np.ndarray, r: Route, expert: ExpertFn, E: int, limit: float = 0.0) -> Diagnostics:
    """All monitoring outputs of one layer step."""
    T, k = r.idx.shape
    rn = expert_output_norms(x, r, expert, limit)
    count = np.bincount(r.idx.reshape(-1), minlength=E)
    norm_mean = np.zeros(E)
    norm_max = np.zeros(E)
    for e in range(E):
        sel = r.idx == e
        if sel.any():
            norm_mean[e] = rn[sel].mean()
            norm_max[e] = rn[sel].max()
    conf = np.take_along_axis(r.s, r.idx, axis=1).mean(axis=1)
    return Diagnostics(count, norm_mean, norm_max, conf, summarise(count, norm_mean, norm_max, conf, T, k), rn)
