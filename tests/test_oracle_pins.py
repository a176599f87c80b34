"""Pins for the fp64 oracle, checked against things other than the oracle itself.

The oracle is the C++ program (``oracle/smoe_oracle.cpp``, exported as ``oracle.*``); the numpy
restatement (``oracle.moe``) is pinned by the same tests: every test below runs once per
implementation (the ``O`` fixture).

The pages print no worked numeric example for the MoE layer, so the oracle is pinned by
brute force on tiny inputs (written as plain loops, not numpy algebra), closed forms,
invariants the pages fix (8 routed + 1 shared expert per token; weights normalised and
scaled by 3; a sigmoid router), special cases that reduce to something simpler, and the bit
layouts of bf16 and fp32 for the input decoders. The last tests plant mistakes — in a copy of the
C++ source, compiled on the fly, and in a copy of the numpy functions — and check these pins
catch them.

Pinned / unpinned, per oracle function:
  bf16_to_f64, f32_to_f64                                 -> hand-built bit patterns decoded by
                                                             the IEEE formula (zeros, subnormals,
                                                             extremes, mantissa tails, infinities)
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
import struct
import types

import numpy as np
import pytest

import oracle

IMPL_NAMES = ["bf16_to_f64", "f32_to_f64", "router_logits", "sigmoid", "select_topk", "normalise", "route",
              "valid_selections", "permute", "silu", "swiglu_hidden", "swiglu_ffn", "moe_sparse", "moe_dense_masked",
              "moe_given_selection", "combine", "Route"]


def _namespace(base, **override):
    ns = types.SimpleNamespace(**{n: getattr(base, n) for n in IMPL_NAMES})
    for name, fn in override.items():
        setattr(ns, name, fn)
    return ns


@pytest.fixture(params=["cpp", "numpy"])
def O(request):
    """The oracle implementation under test: the C++ program or the numpy restatement."""
    return _namespace(oracle if request.param == "cpp" else oracle.moe)


# ------------------------------------------------------------------ input decoders
def _bf16_value(bits: int) -> float:
    """The value of a bf16 bit pattern from the IEEE layout: 1 sign bit, 8 exponent bits (bias
    127), 7 fraction bits."""
    sign = -1.0 if bits >> 15 else 1.0
    e, m = (bits >> 7) & 0xFF, bits & 0x7F
    if e == 0xFF:
        return sign * math.inf if m == 0 else math.nan
    if e == 0:
        return sign * math.ldexp(m, -126 - 7)
    return sign * math.ldexp(128 + m, e - 127 - 7)


def _f32_value(bits: int) -> float:
    """The value of an fp32 bit pattern: 1 sign bit, 8 exponent bits (bias 127), 23 fraction bits."""
    sign = -1.0 if bits >> 31 else 1.0
    e, m = (bits >> 23) & 0xFF, bits & 0x7FFFFF
    if e == 0xFF:
        return sign * math.inf if m == 0 else math.nan
    if e == 0:
        return sign * math.ldexp(m, -126 - 23)
    return sign * math.ldexp((1 << 23) + m, e - 127 - 23)


BF16_CASES = [0x0000, 0x8000, 0x0001, 0x007F, 0x0080, 0x3F80, 0xBF80, 0x3F81, 0x4049, 0xC2F7, 0x7F7F, 0xFF7F,
              0x7F80, 0xFF80]
F32_CASES = [0x00000000, 0x80000000, 0x00000001, 0x007FFFFF, 0x00800000, 0x3F800000, 0x3F800001, 0x40490FDB,
             0xBE4CCCCD, 0x7F7FFFFF, 0xFF7FFFFF, 0x7F800000, 0xFF800000]


def test_bf16_decoder_bit_patterns(O):
    got = O.bf16_to_f64(np.array(BF16_CASES, dtype=np.uint16))
    assert got.dtype == np.float64
    for b, v in zip(BF16_CASES, got.tolist()):
        assert v == _bf16_value(b), hex(b)
        assert math.copysign(1.0, v) == (-1.0 if b >> 15 else 1.0), hex(b)   # the sign of -0 kept
    assert got[2] == 2.0 ** -133 and got[4] == 2.0 ** -126 and got[7] == 1.0 + 2.0 ** -7
    assert got[10] == (2.0 - 2.0 ** -7) * 2.0 ** 127   # the largest finite bf16
    assert math.isnan(O.bf16_to_f64(np.array([0x7FC0], dtype=np.uint16))[0])
    # shape kept; every 16-bit pattern of one exponent decodes to the formula
    grid = np.arange(0x4000, 0x4080, dtype=np.uint16).reshape(8, 16)
    dec = O.bf16_to_f64(grid)
    assert dec.shape == (8, 16)
    assert all(dec.reshape(-1)[i] == _bf16_value(0x4000 + i) for i in range(128))


def test_f32_decoder_bit_patterns(O):
    f = np.array(F32_CASES, dtype=np.uint32).view(np.float32)
    got = O.f32_to_f64(f)
    assert got.dtype == np.float64
    for b, v in zip(F32_CASES, got.tolist()):
        assert v == _f32_value(b), hex(b)
        assert math.copysign(1.0, v) == (-1.0 if b >> 31 else 1.0), hex(b)
    assert got[2] == 2.0 ** -149 and got[6] == 1.0 + 2.0 ** -23
    assert got[9] == (2.0 - 2.0 ** -23) * 2.0 ** 127
    assert got[7] == struct.unpack("<f", struct.pack("<I", 0x40490FDB))[0]


RNG = np.random.default_rng(1234)


def _route_inputs(T, H, E, rng=RNG):
    x = rng.standard_normal((T, H))
    wr = 0.3 * rng.standard_normal((E, H))
    return x, wr


# ------------------------------------------------------------------ router
@pytest.mark.parametrize("E,k", [(6, 2), (10, 3), (7, 7)])
def test_selection_maximises_biased_sum_brute_force(O, E, k):
    x, wr = _route_inputs(40, 8, E)
    bias = 0.05 * RNG.standard_normal(E)
    r = O.route(x, wr, bias, k, 3.0)
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


def test_tie_rule_logit_then_index(O):
    # equal biased scores: the larger raw logit wins, then the smaller index
    bhat = np.array([[0.5, 0.7, 0.7, 0.7, 0.1]])
    logits = np.array([[0.0, 1.0, 2.0, 1.0, 0.0]])
    idx, gap = O.select_topk(bhat, logits, 2)
    assert idx[0].tolist() == [2, 1]
    assert gap[0] == 0.0
    idx, _ = O.select_topk(bhat, logits, 3)
    assert idx[0].tolist() == [2, 1, 3]


def test_sigmoid_closed_forms(O):
    assert O.sigmoid(np.array(0.0)) == 0.5
    assert abs(O.sigmoid(np.array(math.log(3.0))) - 0.75) < 1e-15
    z = np.linspace(-30, 30, 61)
    assert np.allclose(O.sigmoid(-z), 1.0 - O.sigmoid(z), rtol=0, atol=1e-15)


def test_router_logits_brute_force(O):
    x, wr = _route_inputs(3, 5, 4)
    L = O.router_logits(x, wr)
    for t in range(3):
        for e in range(4):
            acc = 0.0
            for h in range(5):
                acc += x[t, h] * wr[e, h]
            assert abs(L[t, e] - acc) < 1e-13


def test_bias_is_selection_only_and_shift_invariant(O):
    x, wr = _route_inputs(50, 16, 12)
    bias = 0.1 * RNG.standard_normal(12)
    r0 = O.route(x, wr, bias, 4, 3.0)
    r1 = O.route(x, wr, bias + 0.375, 4, 3.0)   # exact constant shift (dyadic)
    assert np.array_equal(r0.idx, r1.idx)
    assert np.array_equal(r0.w, r1.w)
    # a huge bias forces an expert in, and its weight still comes from the unbiased score
    big = bias.copy()
    big[5] = 10.0
    r2 = O.route(x, wr, big, 4, 3.0)
    assert np.all((r2.idx == 5).any(axis=1))
    for t in range(50):
        s_sel = r2.s[t, r2.idx[t]]
        assert np.allclose(r2.w[t], 3.0 * s_sel / s_sel.sum(), rtol=1e-15)


def test_weights_sum_to_three_and_positive(O):
    x, wr = _route_inputs(200, 32, 64)
    r = O.route(x, wr, np.zeros(64), 8, 3.0)
    assert np.allclose(r.w.sum(axis=1), 3.0, rtol=0, atol=1e-13)
    assert np.all(r.w > 0)
    # exactly k distinct experts per token
    assert all(len(set(row)) == 8 for row in r.idx.tolist())


def test_all_experts_selected_when_E_equals_k(O):
    x, wr = _route_inputs(10, 8, 5)
    r = O.route(x, wr, np.zeros(5), 5, 3.0)
    for t in range(10):
        assert sorted(r.idx[t].tolist()) == list(range(5))
        s = r.s[t]
        expect = {e: 3.0 * s[e] / s.sum() for e in range(5)}
        for j, e in enumerate(r.idx[t].tolist()):
            assert abs(r.w[t, j] - expect[e]) < 1e-15


def test_near_tie_enumeration(O):
    row = np.array([0.9, 0.8, 0.7, 0.7 + 5e-6, 0.1])
    assert sorted(O.valid_selections(row, 3)) == [(0, 1, 2), (0, 1, 3)]
    row2 = np.array([0.9, 0.8, 0.7, 0.6, 0.1])
    assert O.valid_selections(row2, 3) == [(0, 1, 2)]
    row3 = np.array([0.5, 0.5, 0.5, 0.5])
    assert len(O.valid_selections(row3, 2)) == 6


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
def test_permute_matches_naive_counting_sort(O, T, E, k):
    x, wr = _route_inputs(T, 8, E)
    r = O.route(x, wr, np.zeros(E), k, 3.0)
    counts, offsets, perm_row, row_token = O.permute(r.idx, E)
    c2, o2, p2, rt2 = _naive_permute(r.idx, E)
    assert counts.tolist() == c2 and offsets.tolist() == o2
    assert perm_row.tolist() == p2 and row_token.tolist() == rt2
    assert sorted(perm_row.tolist()) == list(range(T * k))
    assert offsets[-1] == T * k and np.all(np.diff(offsets) >= 0)


# ------------------------------------------------------------------ experts
def test_silu_closed_forms(O):
    assert O.silu(np.array(0.0)) == 0.0
    l3 = math.log(3.0)
    assert abs(O.silu(np.array(l3)) - 0.75 * l3) < 1e-15
    z = np.linspace(-20, 20, 81)
    assert np.allclose(O.silu(-z), O.silu(z) - z, rtol=0, atol=1e-13)


@pytest.mark.parametrize("H,I", [(5, 3), (4, 4)])
def test_swiglu_brute_force_loops(O, H, I):
    x = RNG.standard_normal((2, H))
    Wg, Wu, Wd = RNG.standard_normal((I, H)), RNG.standard_normal((I, H)), RNG.standard_normal((H, I))
    Y = O.swiglu_ffn(x, Wg, Wu, Wd)
    for t in range(2):
        h = []
        for i in range(I):
            g = sum(Wg[i, c] * x[t, c] for c in range(H))
            u = sum(Wu[i, c] * x[t, c] for c in range(H))
            h.append(g / (1.0 + math.exp(-g)) * u)
        for o in range(H):
            y = sum(Wd[o, i] * h[i] for i in range(I))
            assert abs(Y[t, o] - y) < 1e-12


def test_swiglu_identity_weights_closed_form(O):
    l3 = math.log(3.0)
    eye = np.eye(2)
    Y = O.swiglu_ffn(np.array([[l3, 0.0]]), eye, eye, eye)
    assert abs(Y[0, 0] - 0.75 * l3 * l3) < 1e-15 and Y[0, 1] == 0.0


def _tiny_layer(T=12, H=16, E=6, k=2, I=8, seed=7):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, H))
    wr = 0.2 * rng.standard_normal((E, H))
    experts = [tuple(0.2 * rng.standard_normal(s) for s in ((I, H), (I, H), (H, I))) for _ in range(E + 1)]
    return x, wr, experts


def test_single_expert_layer_is_three_F_plus_shared(O):
    x, wr, experts = _tiny_layer(E=1, k=1)
    r = O.route(x, wr, np.zeros(1), 1, 3.0)
    assert np.all(r.w == 3.0)
    out = O.moe_sparse(x, r, lambda e: experts[e], 1)
    expect = 3.0 * O.swiglu_ffn(x, *experts[0]) + O.swiglu_ffn(x, *experts[1])
    assert np.allclose(out, expect, rtol=1e-14, atol=1e-14)


def test_shared_expert_always_applied(O):
    x, wr, experts = _tiny_layer()
    zeroed = [(g, u, np.zeros_like(d)) for g, u, d in experts[:-1]] + [experts[-1]]
    r = O.route(x, wr, np.zeros(6), 2, 3.0)
    out = O.moe_sparse(x, r, lambda e: zeroed[e], 6)
    assert np.array_equal(out, O.swiglu_ffn(x, *experts[-1]))


def test_dense_masked_equals_sparse(O):
    x, wr, experts = _tiny_layer(T=20, E=9, k=3)
    r = O.route(x, wr, 0.01 * np.arange(9), 3, 3.0)
    a = O.moe_sparse(x, r, lambda e: experts[e], 9)
    b = O.moe_dense_masked(x, r, lambda e: experts[e], 9)
    assert np.allclose(a, b, rtol=1e-12, atol=1e-12)


def test_layer_brute_force_loops(O):
    x, wr, experts = _tiny_layer(T=3, H=4, E=4, k=2, I=3)
    r = O.route(x, wr, np.zeros(4), 2, 3.0)
    out = O.moe_sparse(x, r, lambda e: experts[e], 4)

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


def test_given_selection_matches_layer_on_its_own_selection(O):
    x, wr, experts = _tiny_layer()
    r = O.route(x, wr, np.zeros(6), 2, 3.0)
    out = O.moe_sparse(x, r, lambda e: experts[e], 6)
    for t in range(4):
        row = O.moe_given_selection(x[t], r.s[t], r.idx[t].tolist(), lambda e: experts[e], 6, 3.0)
        assert np.allclose(row, out[t], rtol=1e-13, atol=1e-13)


def test_combine_brute_force_loops(O):
    T, k, H = 5, 3, 4
    y = RNG.standard_normal((T * k + T, H))
    perm_row = RNG.permutation(T * k).astype(np.int32)
    w = RNG.random((T, k))
    out = O.combine(y, perm_row, w, T, k)
    for t in range(T):
        for c in range(H):
            acc = y[T * k + t, c]
            for j in range(k):
                acc += w[t, j] * y[perm_row[t * k + j], c]
            assert abs(out[t, c] - acc) < 1e-13


def test_three_matrix_expert_shape_from_parameter_budget(O):
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
def test_swiglu_clamp_brute_force_loops(O, L):
    H, I = 6, 4
    x = 4.0 * RNG.standard_normal((3, H))   # large enough that gate and up cross +-L
    Wg, Wu, Wd = RNG.standard_normal((I, H)), RNG.standard_normal((I, H)), RNG.standard_normal((H, I))
    Y = O.swiglu_ffn(x, Wg, Wu, Wd, limit=L)
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


def test_swiglu_clamp_closed_forms_and_limits(O):
    eye = np.eye(2)
    # gate 10 clamped to 3, up 10 clamped to 3: SiLU(3) * 3 on the diagonal
    Y = O.swiglu_ffn(np.array([[10.0, -10.0]]), eye, eye, eye, limit=3.0)
    s3 = 3.0 / (1.0 + math.exp(-3.0))
    assert abs(Y[0, 0] - s3 * 3.0) < 1e-15
    # gate -10 is not clamped from below: SiLU(-10) * (-3)
    assert abs(Y[0, 1] - (-10.0 / (1.0 + math.exp(10.0))) * -3.0) < 1e-15
    # no clamp for L = 0 and for a limit above every activation
    x, wr, experts = _tiny_layer()
    for e in range(3):
        a = O.swiglu_ffn(x, *experts[e])
        assert np.array_equal(O.swiglu_ffn(x, *experts[e], limit=0.0), a)
        assert np.array_equal(O.swiglu_ffn(x, *experts[e], limit=1e9), a)
    # the layer applies the routed limit to routed experts and the shared limit to the shared one
    r = O.route(x, wr, np.zeros(6), 2, 3.0)
    big = O.moe_sparse(x, r, lambda e: experts[e], 6, limit=1e9, limit_shared=1e9)
    assert np.array_equal(big, O.moe_sparse(x, r, lambda e: experts[e], 6))
    only_shared = O.moe_sparse(x, r, lambda e: experts[e], 6, limit=1e9, limit_shared=0.01)
    assert np.allclose(only_shared - big, O.swiglu_ffn(x, *experts[6], limit=0.01) - O.swiglu_ffn(
        x, *experts[6]), rtol=1e-12, atol=1e-13)


def test_gap_is_kth_minus_next(O):
    bhat = np.array([[0.30, 0.90, 0.55, 0.80, 0.10, 0.56]])
    idx, gap = O.select_topk(bhat, np.zeros_like(bhat), 3)
    assert idx[0].tolist() == [1, 3, 5]
    assert gap[0] == 0.56 - 0.55


# ------------------------------------------------------------------ planted mistakes (numpy restatement)
def _fails(test, O, *args):
    with pytest.raises(AssertionError):
        test(O, *args)


def test_numpy_pins_catch_dropped_scale():
    M = oracle.moe
    _fails(test_weights_sum_to_three_and_positive,
           _namespace(M, route=lambda x, wr, b, k, sc: M.route(x, wr, b, k, 1.0)))


def test_numpy_pins_catch_bias_in_weights():
    M = oracle.moe

    def bad_route(x, wr, bias, k, scale):
        r = M.route(x, wr, bias, k, scale)
        b_sel = np.take_along_axis(r.bhat, r.idx.astype(np.int64), axis=1)
        r.w = M.normalise(b_sel, scale)
        return r
    _fails(test_bias_is_selection_only_and_shift_invariant, _namespace(M, route=bad_route))


def test_numpy_pins_catch_transposed_gate_projection():
    M = oracle.moe
    _fails(test_swiglu_brute_force_loops,
           _namespace(M, swiglu_ffn=lambda X, Wg, Wu, Wd: (M.silu(X @ Wg) * (X @ Wu.T)) @ Wd.T), 4, 4)


def test_numpy_pins_catch_wrong_silu_sign():
    _fails(test_silu_closed_forms, _namespace(oracle.moe, silu=lambda z: z / (1.0 + np.exp(z))))


def test_numpy_pins_catch_gate_clamped_from_below():
    M = oracle.moe

    def bad(X, Wg, Wu, Wd, limit=0.0):
        G, U = X @ Wg.T, X @ Wu.T
        if limit > 0:
            G, U = np.clip(G, -limit, limit), np.clip(U, -limit, limit)
        return (M.silu(G) * U) @ Wd.T
    _fails(test_swiglu_clamp_brute_force_loops, _namespace(M, swiglu_ffn=bad), 0.5)


def test_numpy_pins_catch_truncated_bf16_exponent():
    def bad(bits):   # exponent field read one bit short
        b = np.asarray(bits, dtype=np.uint16) & np.uint16(0xBFFF)
        return oracle.moe.bf16_to_f64(b)
    _fails(test_bf16_decoder_bit_patterns, _namespace(oracle.moe, bf16_to_f64=bad))


# ------------------------------------------------------------------ planted mistakes (C++ program)
# Each case edits one line of a copy of the C++ source, compiles it, swaps it in for the real
# library and checks that the named pin fails.
CPP_PLANTS = {
    "dropped_scale": ("w[t * k + j] = scale * (s_sel[t * k + j] / sum);", "w[t * k + j] = s_sel[t * k + j] / sum;",
                      test_weights_sum_to_three_and_positive, ()),
    "bias_in_weights": ("s_sel[t * k + j] = s[t * E + idx[t * k + j]];",
                        "s_sel[t * k + j] = bhat[t * E + idx[t * k + j]];",
                        test_bias_is_selection_only_and_shift_invariant, ()),
    "tie_rule_larger_index": ("return a < b;", "return a > b;", test_tie_rule_logit_then_index, ()),
    "silu_sign": ("double silu(double z) { return z / (1.0 + std::exp(-z)); }",
                  "double silu(double z) { return z / (1.0 + std::exp(z)); }", test_silu_closed_forms, ()),
    "gate_weights_for_up": ("double u = dot(Wu + i * H, X + r * H, H);", "double u = dot(Wg + i * H, X + r * H, H);",
                            test_swiglu_brute_force_loops, (5, 3)),
    "gate_clamped_from_below": ("g = std::min(g, limit);", "g = std::min(std::max(g, -limit), limit);",
                                test_swiglu_clamp_brute_force_loops, (0.5,)),
    "combine_without_shared": ("double acc = y[(T * k + t) * H + c];", "double acc = 0.0;",
                               test_combine_brute_force_loops, ()),
    "permute_tokens_descending": ("for (int64_t t = 0; t < T; ++t)\n        for (int32_t j = 0; j < k; ++j) {",
                                  "for (int64_t t = T - 1; t >= 0; --t)\n        for (int32_t j = 0; j < k; ++j) {",
                                  test_permute_matches_naive_counting_sort, (13, 9, 3)),
    "dense_mask_ignored": ("wt.push_back(sel ? m : 0.0);", "wt.push_back(sel ? m : 1.0);",
                           test_dense_masked_equals_sparse, ()),
    "shared_expert_dropped": ("swiglu_ffn_rows(x, T, H, wg, wu, wd, I, limit_shared, out);",
                              "for (int64_t q = 0; q < T * H; ++q) out[q] = 0.0;",
                              test_single_expert_layer_is_three_F_plus_shared, ()),
    "bf16_low_half": ("const uint32_t bits = static_cast<uint32_t>(in[i]) << 16;",
                      "const uint32_t bits = static_cast<uint32_t>(in[i]) << 15;",
                      test_bf16_decoder_bit_patterns, ()),
}


@pytest.mark.parametrize("case", sorted(CPP_PLANTS))
def test_cpp_pins_catch_planted_mistake(case, monkeypatch, tmp_path):
    old, new, test, args = CPP_PLANTS[case]
    with open(oracle.cpp.SRC) as f:
        src = f.read()
    assert src.count(old) == 1, f"{case}: the line to plant in is not unique in the source"
    path = tmp_path / "planted.cpp"
    path.write_text(src.replace(old, new))
    planted = oracle.cpp.load(oracle.cpp.build(str(path), str(tmp_path / "libplanted.so")))
    monkeypatch.setattr(oracle.cpp, "_lib", planted)
    with pytest.raises(AssertionError):
        test(_namespace(oracle), *args)
