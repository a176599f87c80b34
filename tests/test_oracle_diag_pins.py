"""Pins for the oracle's monitoring outputs (oracle/diag.py), checked against things other than
the oracle itself: pure-Python loops on a tiny layer, closed forms, invariants, hand-built
statistics, and planted mistakes that these pins must catch.

Pinned per function:
  expert_output_norms  -> pure-Python loops; closed form x^2 sigmoid(x) for 1x1 experts; scaling
  summarise            -> hand-built counts and norms (odd / even active counts, inactive experts)
  diagnostics          -> pure-Python loops for every field; confidence closed form at logit 0
"""
import math
import statistics

import numpy as np
import pytest

import oracle

RNG = np.random.default_rng(99)


def _tiny(T=7, H=4, E=5, k=2, I=3, seed=3):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, H))
    wr = 0.5 * rng.standard_normal((E, H))
    bias = 0.1 * rng.standard_normal(E)
    experts = [tuple(0.5 * rng.standard_normal(s) for s in ((I, H), (I, H), (H, I))) for _ in range(E + 1)]
    return x, wr, bias, experts


def _loops_expert_out(x_row, Wg, Wu, Wd):
    I, H = Wg.shape
    h = []
    for i in range(I):
        g = sum(Wg[i][c] * x_row[c] for c in range(H))
        u = sum(Wu[i][c] * x_row[c] for c in range(H))
        h.append(g / (1.0 + math.exp(-g)) * u)
    return [sum(Wd[o][i] * h[i] for i in range(I)) for o in range(H)]


def test_diagnostics_match_pure_python_loops():
    x, wr, bias, experts = _tiny()
    E, k = 5, 2
    r = oracle.route(x, wr, bias, k, 3.0)
    d = oracle.diagnostics(x, r, lambda e: experts[e], E)
    T = x.shape[0]
    per_expert = {e: [] for e in range(E)}
    conf = []
    for t in range(T):
        sel = [int(e) for e in r.idx[t]]
        s_sel = []
        for e in sel:
            y = _loops_expert_out(list(x[t]), *experts[e])
            per_expert[e].append(math.sqrt(sum(v * v for v in y)))
            logit = sum(wr[e][c] * x[t][c] for c in range(x.shape[1]))
            s_sel.append(1.0 / (1.0 + math.exp(-logit)))
        conf.append(sum(s_sel) / k)
    for e in range(E):
        v = per_expert[e]
        assert d.expert_count[e] == len(v)
        assert math.isclose(d.expert_norm_mean[e], sum(v) / len(v) if v else 0.0, rel_tol=1e-12, abs_tol=1e-14)
        assert math.isclose(d.expert_norm_max[e], max(v) if v else 0.0, rel_tol=1e-12, abs_tol=1e-14)
    assert np.allclose(d.token_confidence, conf, rtol=1e-12, atol=0)
    means = [sum(v) / len(v) for v in per_expert.values() if v]
    med = statistics.median(means)
    expect = [len(means), med, max(means) / med, min(means) / med, sum(conf) / T, min(conf),
              max(len(v) for v in per_expert.values()) / (T * k / E),
              max(max(v) for v in per_expert.values() if v)]
    assert np.allclose(d.summary, expect, rtol=1e-12, atol=0)


def test_norm_closed_form_for_one_by_one_experts():
    # E = k = 1, H = I = 1, all weights 1: F(x) = SiLU(x) x = x^2 sigmoid(x); at x = ln 3, 0.75 ln^2 3
    l3 = math.log(3.0)
    x = np.array([[l3], [-l3]])
    r = oracle.route(x, np.zeros((1, 1)), np.zeros(1), 1, 3.0)
    one = (np.ones((1, 1)), np.ones((1, 1)), np.ones((1, 1)))
    d = oracle.diagnostics(x, r, lambda e: one, 1)
    assert abs(d.row_norm[0, 0] - 0.75 * l3 * l3) < 1e-14
    assert abs(d.row_norm[1, 0] - 0.25 * l3 * l3) < 1e-14
    assert abs(d.expert_norm_mean[0] - 0.5 * l3 * l3) < 1e-14
    # router weights 0: every logit is 0, every score 1/2, so every confidence is exactly 1/2
    assert np.all(d.token_confidence == 0.5)


def test_scaling_the_down_projection_scales_norms_not_ratios():
    x, wr, bias, experts = _tiny(T=11, E=6)
    r = oracle.route(x, wr, bias, 2, 3.0)
    a = oracle.diagnostics(x, r, lambda e: experts[e], 6)
    b = oracle.diagnostics(x, r, lambda e: (experts[e][0], experts[e][1], 2.5 * experts[e][2]), 6)
    assert np.allclose(b.expert_norm_mean, 2.5 * a.expert_norm_mean, rtol=1e-12)
    assert np.allclose(b.row_norm, 2.5 * a.row_norm, rtol=1e-12)
    assert np.allclose(b.summary[2:4], a.summary[2:4], rtol=1e-12)
    assert np.array_equal(a.expert_count, b.expert_count)
    assert a.expert_count.sum() == 11 * 2


def test_summary_hand_built_statistics():
    conf = np.array([0.25, 0.5, 0.75, 1.0])
    # four active experts, even count: median = (2 + 3) / 2
    s = oracle.summarise(np.array([1, 2, 3, 2]), np.array([1.0, 2.0, 3.0, 10.0]), np.array([1.0, 4.0, 5.0, 12.0]),
                         conf, T=4, k=2)
    assert np.allclose(s, [4, 2.5, 4.0, 0.4, 0.625, 0.25, 3 / 2, 12.0])
    # an expert without tokens is left out of the median and the ratios
    s = oracle.summarise(np.array([0, 3, 2, 3]), np.array([100.0, 1.0, 2.0, 4.0]), np.array([0.0, 1, 2, 4]),
                         conf, T=4, k=2)
    assert np.allclose(s, [3, 2.0, 2.0, 0.5, 0.625, 0.25, 3 / 2, 4.0])


# ------------------------------------------------------------------ planted mistakes
def test_pins_catch_squared_norm(monkeypatch):
    def bad(x, r, expert, limit=0.0):
        T, k = r.idx.shape
        n = np.zeros((T, k))
        for e in np.unique(r.idx):
            rows, slots = np.nonzero(r.idx == e)
            y = oracle.swiglu_ffn(x[rows], *expert(int(e)), limit=limit)
            n[rows, slots] = np.sum(y * y, axis=1)
        return n
    monkeypatch.setattr(oracle.diag, "expert_output_norms", bad)
    with pytest.raises(AssertionError):
        test_norm_closed_form_for_one_by_one_experts()


def test_pins_catch_median_over_all_experts(monkeypatch):
    def bad(count, norm_mean, norm_max, conf, T, k):
        med = float(np.median(norm_mean))
        return np.array([int((count > 0).sum()), med, norm_mean.max() / med, norm_mean.min() / med, conf.mean(),
                         conf.min(), count.max() / (T * k / count.shape[0]), norm_max.max()])
    monkeypatch.setattr(oracle, "summarise", bad)
    with pytest.raises(AssertionError):
        test_summary_hand_built_statistics()


def test_pins_catch_confidence_from_biased_scores(monkeypatch):
    real = oracle.diag.diagnostics

    def bad(x, r, expert, E, limit=0.0):
        d = real(x, r, expert, E, limit)
        d.token_confidence = np.take_along_axis(r.bhat, r.idx, axis=1).mean(axis=1)
        return d
    monkeypatch.setattr(oracle, "diagnostics", bad)
    with pytest.raises(AssertionError):
        test_diagnostics_match_pure_python_loops()
