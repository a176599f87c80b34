"""The C++ oracle against the numpy restatement of the same layer (two independent codes from the
same reading of the pages), and the C++ oracle's independence from its thread count.

Agreement to 1e-12 (relative to the largest output) means neither carries a mistake the other
lacks: the two differ only in summation order (sequential loops against BLAS).
"""
import numpy as np
import pytest

import oracle
import synth

M = oracle.moe
REL = 1e-12


def _rel(a, b):
    return np.abs(a - b).max() / max(np.abs(b).max(), 1e-300)


def _random_layer(T, H, E, k, I, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, H))
    wr = 0.3 * rng.standard_normal((E, H))
    bias = 0.05 * rng.standard_normal(E)
    experts = [tuple(0.2 * rng.standard_normal(s) for s in ((I, H), (I, H), (H, I))) for _ in range(E + 1)]
    return x, wr, bias, experts


@pytest.mark.parametrize("T,H,E,k,I,limit", [(1, 8, 4, 2, 4, 0.0), (37, 32, 12, 3, 16, 0.0), (64, 64, 32, 4, 24, 0.0),
                                             (50, 48, 10, 10, 8, 0.0), (40, 32, 16, 4, 16, 0.7)])
def test_layer_agrees_with_numpy(T, H, E, k, I, limit):
    x, wr, bias, experts = _random_layer(T, H, E, k, I, seed=T * 7 + E)
    rc, rn = oracle.route(x, wr, bias, k, 3.0), M.route(x, wr, bias, k, 3.0)
    assert _rel(rc.logits, rn.logits) <= REL
    assert np.array_equal(rc.idx, rn.idx)
    assert _rel(rc.w, rn.w) <= REL and _rel(rc.s, rn.s) <= REL
    fin = np.isfinite(rn.gap)
    assert np.array_equal(np.isfinite(rc.gap), fin) and np.allclose(rc.gap[fin], rn.gap[fin], rtol=0, atol=1e-15)
    for a, b in zip(oracle.permute(rc.idx, E), M.permute(rn.idx, E)):
        assert np.array_equal(a, b)
    ex = lambda e: experts[e]   # noqa: E731
    lim = dict(limit=limit, limit_shared=limit / 2)
    sp = oracle.moe_sparse(x, rc, ex, E, **lim)
    assert _rel(sp, M.moe_sparse(x, rn, ex, E, **lim)) <= REL
    dn = oracle.moe_dense_masked(x, rc, ex, E, **lim)
    assert _rel(dn, M.moe_dense_masked(x, rn, ex, E, **lim)) <= REL
    assert np.array_equal(sp, dn)   # same terms in the same order; masked terms are exact zeros
    row = oracle.moe_given_selection(x[0], rc.s[0], rc.idx[0].tolist(), ex, E, 3.0, **lim)
    assert _rel(row, M.moe_given_selection(x[0], rn.s[0], rn.idx[0].tolist(), ex, E, 3.0, **lim)) <= REL
    y = np.random.default_rng(T).standard_normal((T * k + T, H))
    pr = oracle.permute(rc.idx, E)[2]
    assert _rel(oracle.combine(y, pr, rc.w, T, k), M.combine(y, pr, rn.w, T, k)) <= REL
    for t in range(min(T, 5)):
        assert sorted(oracle.valid_selections(rc.bhat[t], k)) == sorted(M.valid_selections(rn.bhat[t], k))


def test_tiny_workload_dense_masked_agrees_with_numpy():
    """The tiny layer configuration (T=64, H=512, E=32, k=4, I=128) on its seeded inputs."""
    w = synth.WORKLOADS["tiny"]
    x = oracle.bf16_to_f64(synth.host_x(w))
    assert np.array_equal(x, M.bf16_to_f64(synth.host_x(w)))
    wr = oracle.f32_to_f64(synth.host_w_router(w))
    bias = synth.host_bias(w).astype(np.float64)
    experts = {e: tuple(oracle.bf16_to_f64(a) for a in synth.host_expert(w, e)) for e in range(w.E + 1)}
    rc, rn = oracle.route(x, wr, bias, w.k, w.route_scale), M.route(x, wr, bias, w.k, w.route_scale)
    assert np.array_equal(rc.idx, rn.idx)
    a = oracle.moe_dense_masked(x, rc, lambda e: experts[e], w.E)
    assert _rel(a, M.moe_dense_masked(x, rn, lambda e: experts[e], w.E)) <= REL


def test_decode_workload_sample_agrees_with_numpy():
    """The Step-shape decode batch: router on all 64 tokens, the sparse layer on 3 of them."""
    w = synth.WORKLOADS["decode"]
    x = oracle.bf16_to_f64(synth.host_x(w))
    wr = oracle.f32_to_f64(synth.host_w_router(w))
    bias = synth.host_bias(w).astype(np.float64)
    rc, rn = oracle.route(x, wr, bias, w.k, w.route_scale), M.route(x, wr, bias, w.k, w.route_scale)
    assert np.array_equal(rc.idx, rn.idx) and _rel(rc.logits, rn.logits) <= REL
    rows = [0, 31, 63]
    cache = {}

    def ex(e):
        if e not in cache:
            cache[e] = tuple(oracle.bf16_to_f64(a) for a in synth.host_expert(w, e))
        return cache[e]
    sub_c = oracle.Route(*(getattr(rc, f)[rows] for f in ("logits", "s", "bhat", "idx", "w", "gap")))
    sub_n = oracle.Route(*(getattr(rn, f)[rows] for f in ("logits", "s", "bhat", "idx", "w", "gap")))
    assert _rel(oracle.moe_sparse(x[rows], sub_c, ex, w.E), M.moe_sparse(x[rows], sub_n, ex, w.E)) <= REL


def test_results_do_not_depend_on_the_thread_count():
    x, wr, bias, experts = _random_layer(33, 40, 9, 3, 12, seed=5)
    outs = []
    try:
        for n in (1, 3, 0):
            oracle.cpp.set_threads(n)
            r = oracle.route(x, wr, bias, 3, 3.0)
            outs.append((r.logits, r.idx, oracle.moe_sparse(x, r, lambda e: experts[e], 9)))
    finally:
        oracle.cpp.set_threads(0)
    for o in outs[1:]:
        assert all(np.array_equal(a, b) for a, b in zip(o, outs[0]))


def test_bad_inputs_are_refused():
    idx = np.array([[0, 5]], dtype=np.int32)
    with pytest.raises(ValueError):
        oracle.permute(idx, 4)   # expert id 5 of 4
    with pytest.raises(ValueError):
        oracle.combine(np.zeros((3, 2)), np.array([0, 7], dtype=np.int32), np.ones((1, 2)), 1, 2)


def test_forward_timed_matches_the_layer():
    x, wr, bias, experts = _random_layer(12, 16, 6, 2, 8, seed=9)
    out, sec = oracle.cpp.forward_timed(x, wr, bias, 2, 3.0, lambda e: experts[e], 6, repeats=3)
    r = oracle.route(x, wr, bias, 2, 3.0)
    assert np.array_equal(out, oracle.moe_sparse(x, r, lambda e: experts[e], 6))
    assert sec > 0.0
