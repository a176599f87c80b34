"""Writes tests/golden/zipf_bias.json: the bias strength beta of the skewed-routing workload.

Recipe (the pages give none; this is the stated reading for the skewed workload):
  * experts get popularity ranks r = 1..288 from a seeded hash (synth.zipf_ranks);
  * the 16 lowest-ranked experts get bias -100 (never selected: dead experts);
  * live experts get bias_e = -beta * ln(r_e);
  * beta is found by bisection so that the log-log slope of the realised per-expert token
    counts against rank, over live ranks that are neither empty nor saturated (count < T),
    is -1.2 (Zipf s = 1.2). Selection is the fp64 oracle's router on the workload's seeded x.

Only the oracle computes here (router logits, sigmoid, top-k). Run from the repo root:
    python tests/golden/make_zipf_bias.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
import synth  # noqa: E402

TARGET_SLOPE = -1.2


def realised(w, s, L, beta):
    bias = synth.zipf_bias(w, beta).astype(np.float64)
    idx, _ = oracle.select_topk(s + bias[None, :], L, w.k)
    counts = np.bincount(idx.reshape(-1), minlength=w.E)
    ranks = synth.zipf_ranks(w)
    by_rank = np.zeros(w.E, dtype=np.int64)
    by_rank[ranks - 1] = counts
    live = np.arange(1, w.E - synth.ZIPF_DEAD + 1)
    c = by_rank[: len(live)]
    use = (c > 0) & (c < w.T)
    slope = np.polyfit(np.log(live[use]), np.log(c[use]), 1)[0]
    return slope, by_rank


def main():
    w = synth.WORKLOADS["skewed"]
    x = oracle.bf16_to_f64(synth.host_x(w))
    wr = oracle.f32_to_f64(synth.host_w_router(w))
    L = oracle.router_logits(x, wr)
    s = oracle.sigmoid(L)
    lo, hi = 0.0, 1.0
    while realised(w, s, L, hi)[0] > TARGET_SLOPE:
        hi *= 2.0
    for _ in range(40):
        mid = 0.5 * (lo + hi)
        if realised(w, s, L, mid)[0] > TARGET_SLOPE:
            lo = mid
        else:
            hi = mid
    beta = float(np.float32(0.5 * (lo + hi)))
    slope, by_rank = realised(w, s, L, beta)
    out = {
        "beta": beta,
        "target_slope": TARGET_SLOPE,
        "realised_slope": float(slope),
        "dead_experts": synth.ZIPF_DEAD,
        "T": w.T,
        "counts_by_rank": by_rank.tolist(),
        "recipe": "bias_e = -beta*ln(rank_e) for live ranks, -100 for the 16 lowest; beta by bisection on the "
                  "realised log-log slope of counts vs rank (fp64 oracle router, seeded x).",
    }
    with open(os.path.join(HERE, "zipf_bias.json"), "w") as f:
        json.dump(out, f, indent=1)
    print(f"beta={beta:.6f} slope={slope:.4f} top counts={by_rank[:8].tolist()} "
          f"empty live={int((by_rank[:w.E - synth.ZIPF_DEAD] == 0).sum())}")


if __name__ == "__main__":
    main()
