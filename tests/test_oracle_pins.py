"""Pins for the fp64 oracle, checked against things other than the oracle itself.

The pages print no worked numeric example for the MoE layer, so the oracle is pinned by
brute force on tiny inputs (written as plain loops, not numpy algebra), closed forms,
invariants the pages fix (8 routed + 1 shared expert per token; weights normalised and
scaled by 3; a sigmoid router), and special cases that reduce to something simpler.
The last tests plant mistakes in a copy of the oracle and check these pins catch them.

Pinned / unpinned, per oracle function:
  router_logits, sigmoid, select_topk, normalise, route  -> brute force + closed forms + invariants
  valid_selections                                        -> hand-built tie rows
  permute                                                 -> pure-Python counting sort
  silu, swiglu_ffn, swiglu_hidden                         -> closed forms + pure-Python loops
  moe_sparse, moe_dense_masked, moe_given_selection       -> special cases (E=k=1, zero W_d,
                                                             dense == sparse) + loop brute force
  combine                                                 -> pure-Python loops
Absolute output values at the Step shape: no page value exists -> checked only through the
pins above ("parity unpinned" beyond them).
"""
import itertools
import math

import numpy as np
import pytest

import oracle

RNG = np.random.default_rng(1234)


def _route_inputs(T, H, E, rng=RNG):
    x = rng.standard_normal((T, H))
    wr = 0.3 * rng.standard_normal((E, H))
    return x, wr


# ------------------------------------------------------------------ router
@pytest.mark.parametrize("E,k", [(6, 2), (10, 3), (7, 7)])
def test_selection_maximises_biased_sum_brute_force(E, k):
    x, wr = _route_inputs(40, 8, E)
    bias = 0.05 * RNG.standard_normal(E)
    r = oracle.route(x, wr, bias, k, 3.0)
    for t in range(x.shape[0]):
        # brute force over every k-subset, with plain loops
        best, best_sum = None, -math.inf
        for S in itertools.combinations(range(E), k):
            ssum = 0.0
            for e in S:
                dot = 0.0
                for h in range(x.shape[1]):
                    dot += x[t, h] * wr[e, h]
                ssum += 1.0 / (1.0 + math.exp(-dot)) + bias[e]
            if ssum > best_sum:
                best, best_sum = S, ssum
        assert set(r.idx[t].tolist()) == set(best)
        # descending order by biased score
        b = r.bhat[t, r.idx[t]]
        assert np.all(np.diff(b) <= 0)


def test_tie_rule_logit_then_index():
    # equal biased scores: the larger raw logit wins, then the smaller index
    bhat = np.array([[0.5, 0.7, 0.7, 0.7, 0.1]])
    logits = np.array([[0.0, 1.0, 2.0, 1.0, 0.0]])
    idx, gap = oracle.select_topk(bhat, logits, 2)
    assert idx[0].tolist() == [2, 1]
    assert gap[0] == 0.0
    idx, _ = oracle.select_topk(bhat, logits, 3)
    assert idx[0].tolist() == [2, 1, 3]


def test_sigmoid_closed_forms():
    assert oracle.sigmoid(np.array(0.0)) == 0.5
    assert abs(oracle.sigmoid(np.array(math.log(3.0))) - 0.75) < 1e-15
    z = np.linspace(-30, 30, 61)
    assert np.allclose(oracle.sigmoid(-z), 1.0 - oracle.sigmoid(z), rtol=0, atol=1e-15)


def test_router_logits_brute_force():
    x, wr = _route_inputs(3, 5, 4)
    L = oracle.router_logits(x, wr)
    for t in range(3):
        for e in range(4):
            acc = 0.0
            for h in range(5):
                acc += x[t, h] * wr[e, h]
            assert abs(L[t, e] - acc) < 1e-13


def test_bias_is_selection_only_and_shift_invariant():
    x, wr = _route_inputs(50, 16, 12)
    bias = 0.1 * RNG.standard_normal(12)
    r0 = oracle.route(x, wr, bias, 4, 3.0)
    r1 = oracle.route(x, wr, bias + 0.375, 4, 3.0)   # exact constant shift (dyadic)
    assert np.array_equal(r0.idx, r1.idx)
    assert np.array_equal(r0.w, r1.w)
    # a huge bias forces an expert in, and its weight still comes from the unbiased score
    big = bias.copy()
    big[5] = 10.0
    r2 = oracle.route(x, wr, big, 4, 3.0)
    assert np.all((r2.idx == 5).any(axis=1))
    for t in range(50):
        s_sel = r2.s[t, r2.idx[t]]
        assert np.allclose(r2.w[t], 3.0 * s_sel / s_sel.sum(), rtol=1e-15)


def test_weights_sum_to_three_and_positive():
    x, wr = _route_inputs(200, 32, 64)
    r = oracle.route(x, wr, np.zeros(64), 8, 3.0)
    assert np.allclose(r.w.sum(axis=1), 3.0, rtol=0, atol=1e-13)
    assert np.all(r.w > 0)
    # exactly k distinct experts per token
    assert all(len(set(row)) == 8 for row in r.idx.tolist())


def test_all_experts_selected_when_E_equals_k():
    x, wr = _route_inputs(10, 8, 5)
    r = oracle.route(x, wr, np.zeros(5), 5, 3.0)
    for t in range(10):
        assert sorted(r.idx[t].tolist()) == list(range(5))
        s = r.s[t]
        expect = {e: 3.0 * s[e] / s.sum() for e in range(5)}
        for j, e in enumerate(r.idx[t].tolist()):
            assert abs(r.w[t, j] - expect[e]) < 1e-15


def test_near_tie_enumeration():
    row = np.array([0.9, 0.8, 0.7, 0.7 + 5e-6, 0.1])
    assert sorted(oracle.valid_selections(row, 3)) == [(0, 1, 2), (0, 1, 3)]
    row2 = np.array([0.9, 0.8, 0.7, 0.6, 0.1])
    assert oracle.valid_selections(row2, 3) == [(0, 1, 2)]
    row3 = np.array([0.5, 0.5, 0.5, 0.5])
    assert len(oracle.valid_selections(row3, 2)) == 6


# ------------------------------------------------------------------ permute
def _naive_permute(idx, E):
    T, k = idx.shape
    rows = []
    for e in range(E):
        for t in range(T):
            for j in range(k):
                if idx[t, j] == e:
                    rows.append((t, j))
    counts = [sum(1 for t in range(T) for j in range(k) if idx[t, j] == e) for e in range(E)]
    offsets = [0]
    for c in counts:
        offsets.append(offsets[-1] + c)
    perm_row = [0] * (T * k)
    row_token = [0] * (T * k)
    for r, (t, j) in enumerate(rows):
        perm_row[t * k + j] = r
        row_token[r] = t
    return counts, offsets, perm_row, row_token


@pytest.mark.parametrize("T,E,k", [(1, 4, 2), (13, 9, 3), (64, 32, 4)])
def test_permute_matches_naive_counting_sort(T, E, k):
    x, wr = _route_inputs(T, 8, E)
    r = oracle.route(x, wr, np.zeros(E), k, 3.0)
    counts, offsets, perm_row, row_token = oracle.permute(r.idx, E)
    c2, o2, p2, rt2 = _naive_permute(r.idx, E)
    assert counts.tolist() == c2 and offsets.tolist() == o2
    assert perm_row.tolist() == p2 and row_token.tolist() == rt2
    assert sorted(perm_row.tolist()) == list(range(T * k))
    assert offsets[-1] == T * k and np.all(np.diff(offsets) >= 0)


# ------------------------------------------------------------------ experts
def test_silu_closed_forms():
    assert oracle.silu(np.array(0.0)) == 0.0
    l3 = math.log(3.0)
    assert abs(oracle.silu(np.array(l3)) - 0.75 * l3) < 1e-15
    z = np.linspace(-20, 20, 81)
    assert np.allclose(oracle.silu(-z), oracle.silu(z) - z, rtol=0, atol=1e-13)


@pytest.mark.parametrize("H,I", [(5, 3), (4, 4)])
def test_swiglu_brute_force_loops(H, I):
    x = RNG.standard_normal((2, H))
    Wg, Wu, Wd = RNG.standard_normal((I, H)), RNG.standard_normal((I, H)), RNG.standard_normal((H, I))
    Y = oracle.swiglu_ffn(x, Wg, Wu, Wd)
    for t in range(2):
        h = []
        for i in range(I):
            g = sum(Wg[i, c] * x[t, c] for c in range(H))
            u = sum(Wu[i, c] * x[t, c] for c in range(H))
            h.append(g / (1.0 + math.exp(-g)) * u)
        for o in range(H):
            y = sum(Wd[o, i] * h[i] for i in range(I))
            assert abs(Y[t, o] - y) < 1e-12


def test_swiglu_identity_weights_closed_form():
    l3 = math.log(3.0)
    eye = np.eye(2)
    Y = oracle.swiglu_ffn(np.array([[l3, 0.0]]), eye, eye, eye)
    assert abs(Y[0, 0] - 0.75 * l3 * l3) < 1e-15 and Y[0, 1] == 0.0


def _tiny_layer(T=12, H=16, E=6, k=2, I=8, seed=7):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, H))
    wr = 0.2 * rng.standard_normal((E, H))
    experts = [tuple(0.2 * rng.standard_normal(s) for s in ((I, H), (I, H), (H, I))) for _ in range(E + 1)]
    return x, wr, experts


def test_single_expert_layer_is_three_F_plus_shared():
    x, wr, experts = _tiny_layer(E=1, k=1)
    r = oracle.route(x, wr, np.zeros(1), 1, 3.0)
    assert np.all(r.w == 3.0)
    out = oracle.moe_sparse(x, r, lambda e: experts[e], 1)
    expect = 3.0 * oracle.swiglu_ffn(x, *experts[0]) + oracle.swiglu_ffn(x, *experts[1])
    assert np.allclose(out, expect, rtol=1e-14, atol=1e-14)


def test_shared_expert_always_applied():
    x, wr, experts = _tiny_layer()
    zeroed = [(g, u, np.zeros_like(d)) for g, u, d in experts[:-1]] + [experts[-1]]
    r = oracle.route(x, wr, np.zeros(6), 2, 3.0)
    out = oracle.moe_sparse(x, r, lambda e: zeroed[e], 6)
    assert np.array_equal(out, oracle.swiglu_ffn(x, *experts[-1]))


def test_dense_masked_equals_sparse():
    x, wr, experts = _tiny_layer(T=20, E=9, k=3)
    r = oracle.route(x, wr, 0.01 * np.arange(9), 3, 3.0)
    a = oracle.moe_sparse(x, r, lambda e: experts[e], 9)
    b = oracle.moe_dense_masked(x, r, lambda e: experts[e], 9)
    assert np.allclose(a, b, rtol=1e-12, atol=1e-12)


def test_layer_brute_force_loops():
    x, wr, experts = _tiny_layer(T=3, H=4, E=4, k=2, I=3)
    r = oracle.route(x, wr, np.zeros(4), 2, 3.0)
    out = oracle.moe_sparse(x, r, lambda e: experts[e], 4)

    def F(e, xt):
        Wg, Wu, Wd = experts[e]
        h = [(lambda g: g / (1 + math.exp(-g)))(sum(Wg[i, c] * xt[c] for c in range(4))) *
             sum(Wu[i, c] * xt[c] for c in range(4)) for i in range(3)]
        return [sum(Wd[o, i] * h[i] for i in range(3)) for o in range(4)]

    for t in range(3):
        logits = [sum(x[t, c] * wr[e, c] for c in range(4)) for e in range(4)]
        s = [1 / (1 + math.exp(-v)) for v in logits]
        top = sorted(range(4), key=lambda e: -s[e])[:2]
        tot = s[top[0]] + s[top[1]]
        y = F(4, x[t])
        for e in top:
            fe = F(e, x[t])
            y = [a + 3.0 * s[e] / tot * b for a, b in zip(y, fe)]
        assert np.allclose(out[t], y, rtol=1e-12, atol=1e-12)


def test_given_selection_matches_layer_on_its_own_selection():
    x, wr, experts = _tiny_layer()
    r = oracle.route(x, wr, np.zeros(6), 2, 3.0)
    out = oracle.moe_sparse(x, r, lambda e: experts[e], 6)
    for t in range(4):
        row = oracle.moe_given_selection(x[t], r.s[t], r.idx[t].tolist(), lambda e: experts[e], 6, 3.0)
        assert np.allclose(row, out[t], rtol=1e-13, atol=1e-13)


def test_combine_brute_force_loops():
    T, k, H = 5, 3, 4
    y = RNG.standard_normal((T * k + T, H))
    perm_row = RNG.permutation(T * k).astype(np.int32)
    w = RNG.random((T, k))
    out = oracle.combine(y, perm_row, w, T, k)
    for t in range(T):
        for c in range(H):
            acc = y[T * k + t, c]
            for j in range(k):
                acc += w[t, j] * y[perm_row[t * k + j], c]
            assert abs(out[t, c] - acc) < 1e-13


def test_three_matrix_expert_shape_from_parameter_budget():
    # 42 MoE layers x (288 routed + 1 shared) experts of H=4096, I=1280 must fit the stated
    # 196B total; a 3-matrix (gate, up, down) expert gives ~191B, a 2-matrix one only ~127B.
    H, I, E, layers = 4096, 1280, 288, 42
    three = 3 * H * I * (E + 1) * layers
    two = 2 * H * I * (E + 1) * layers
    assert 185e9 < three < 196e9
    assert two < 130e9
    # active per token: 8 routed + 1 shared experts within the stated 11B active
    assert 3 * H * I * 9 * layers < 11e9


@pytest.mark.parametrize("L", [0.5, 2.0, 7.0])
def test_swiglu_clamp_brute_force_loops(L):
    H, I = 6, 4
    x = 4.0 * RNG.standard_normal((3, H))   # large enough that gate and up cross +-L
    Wg, Wu, Wd = RNG.standard_normal((I, H)), RNG.standard_normal((I, H)), RNG.standard_normal((H, I))
    Y = oracle.swiglu_ffn(x, Wg, Wu, Wd, limit=L)
    crossed = 0
    for t in range(3):
        h = []
        for i in range(I):
            g = sum(Wg[i, c] * x[t, c] for c in range(H))
            u = sum(Wu[i, c] * x[t, c] for c in range(H))
            crossed += (g > L) + (abs(u) > L) + (g < -L)
            g = g if g < L else L
            u = -L if u < -L else (L if u > L else u)
            h.append(g / (1.0 + math.exp(-g)) * u)
        for o in range(H):
            assert abs(Y[t, o] - sum(Wd[o, i] * h[i] for i in range(I))) < 1e-11
    assert crossed > 0


def test_swiglu_clamp_closed_forms_and_limits():
    eye = np.eye(2)
    # gate 10 clamped to 3, up 10 clamped to 3: SiLU(3) * 3 on the diagonal
    Y = oracle.swiglu_ffn(np.array([[10.0, -10.0]]), eye, eye, eye, limit=3.0)
    s3 = 3.0 / (1.0 + math.exp(-3.0))
    assert abs(Y[0, 0] - s3 * 3.0) < 1e-15
    # gate -10 is not clamped from below: SiLU(-10) * (-3)
    assert abs(Y[0, 1] - (-10.0 / (1.0 + math.exp(10.0))) * -3.0) < 1e-15
    # no clamp for L = 0 and for a limit above every activation
    x, wr, experts = _tiny_layer()
    for e in range(3):
        a = oracle.swiglu_ffn(x, *experts[e])
        assert np.array_equal(oracle.swiglu_ffn(x, *experts[e], limit=0.0), a)
        assert np.array_equal(oracle.swiglu_ffn(x, *experts[e], limit=1e9), a)
    # the layer applies the routed limit to routed experts and the shared limit to the shared one
    r = oracle.route(x, wr, np.zeros(6), 2, 3.0)
    big = oracle.moe_sparse(x, r, lambda e: experts[e], 6, limit=1e9, limit_shared=1e9)
    assert np.array_equal(big, oracle.moe_sparse(x, r, lambda e: experts[e], 6))
    only_shared = oracle.moe_sparse(x, r, lambda e: experts[e], 6, limit=1e9, limit_shared=0.01)
    assert np.allclose(only_shared - big, oracle.swiglu_ffn(x, *experts[6], limit=0.01) - oracle.swiglu_ffn(
        x, *experts[6]), rtol=1e-12, atol=1e-13)


# ------------------------------------------------------------------ planted mistakes
def _pins_fail(monkeypatch, name, fn, test, *args):
    monkeypatch.setattr(oracle, name, fn)
    with pytest.raises(AssertionError):
        test(*args)


def test_pins_catch_dropped_scale(monkeypatch):
    _pins_fail(monkeypatch, "route",
               lambda x, wr, b, k, sc: oracle.moe.route(x, wr, b, k, 1.0),
               test_weights_sum_to_three_and_positive)


def test_pins_catch_bias_in_weights(monkeypatch):
    def bad_route(x, wr, bias, k, scale):
        r = oracle.moe.route(x, wr, bias, k, scale)
        b_sel = np.take_along_axis(r.bhat, r.idx.astype(np.int64), axis=1)
        r.w = oracle.moe.normalise(b_sel, scale)
        return r
    _pins_fail(monkeypatch, "route", bad_route, test_bias_is_selection_only_and_shift_invariant)


def test_pins_catch_transposed_gate_projection(monkeypatch):
    monkeypatch.setattr(oracle, "swiglu_ffn",
                        lambda X, Wg, Wu, Wd: (oracle.moe.silu(X @ Wg) * (X @ Wu.T)) @ Wd.T)
    with pytest.raises(AssertionError):
        test_swiglu_brute_force_loops(4, 4)


def test_pins_catch_wrong_silu_sign(monkeypatch):
    monkeypatch.setattr(oracle, "silu", lambda z: z / (1.0 + np.exp(z)))
    with pytest.raises(AssertionError):
        test_silu_closed_forms()


def test_pins_catch_gate_clamped_from_below(monkeypatch):
    def bad(X, Wg, Wu, Wd, limit=0.0):
        G, U = X @ Wg.T, X @ Wu.T
        if limit > 0:
            G, U = np.clip(G, -limit, limit), np.clip(U, -limit, limit)
        return (oracle.moe.silu(G) * U) @ Wd.T
    monkeypatch.setattr(oracle, "swiglu_ffn", bad)
    with pytest.raises(AssertionError):
        test_swiglu_clamp_brute_force_loops(0.5)
