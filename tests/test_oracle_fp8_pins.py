"""Pins for the FP8 (e4m3) oracle (oracle/fp8.py), against things other than the oracle itself:
the e4m3 format built from its bit definition, brute-force nearest-value search, closed forms
of the scaling, and special cases where quantisation is exact. Planted mistakes must fail.

Pinned per function:
  e4m3_round / e4m3_code / e4m3_decode -> the 256 codes built from the bit layout; brute-force
                                          nearest-with-ties-to-even over random and tie inputs
  quantize_rows                        -> closed forms (row maximum -> +-448, zero rows, scale)
  round_bf16                           -> bf16 bit-level rounding of hand-picked fp32 values
  swiglu_ffn_fp8 / moe_sparse_fp8      -> exact equality with the fp64 gate/up products when every
                                          quantity is already on the e4m3 grid with power-of-two
                                          scales; closeness to the fp64 layer otherwise
"""
import math

import numpy as np
import pytest

import oracle

RNG = np.random.default_rng(8)


def _all_finite_e4m3():
    """Every finite e4m3 value with its code, from the bit layout (independent of the oracle)."""
    vals, codes = [], []
    for c in range(256):
        s, e, m = c >> 7, (c >> 3) & 15, c & 7
        if e == 15 and m == 7:
            continue   # NaN
        mag = m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
        vals.append(-mag if s else mag)
        codes.append(c)
    return np.array(vals), np.array(codes, dtype=np.uint8)


def _brute_nearest(x, grid, codes):
    """Nearest grid value; on an exact tie the even code (mantissa lsb 0); saturating."""
    out = np.empty_like(x)
    pos = np.sort(np.unique(np.abs(grid)))
    for i, v in enumerate(x):
        mag = min(abs(v), 448.0)
        d = np.abs(pos - mag)
        best = np.nonzero(d == d.min())[0]
        if len(best) > 1:
            cands = pos[best]
            cc = [codes[np.nonzero(grid == c)[0][0]] for c in cands]
            pick = cands[[int(c) & 1 == 0 for c in cc].index(True)]
        else:
            pick = pos[best[0]]
        out[i] = math.copysign(pick, v)
    return out


def test_codes_roundtrip_and_match_the_bit_layout():
    grid, codes = _all_finite_e4m3()
    assert grid.max() == 448.0 and np.min(np.abs(grid[grid != 0])) == 2.0 ** -9
    assert np.array_equal(oracle.e4m3_decode(codes), grid)
    assert np.array_equal(oracle.e4m3_round(grid), grid)
    # every code except the negative zero and NaNs round-trips through the value
    keep = codes != 0x80
    assert np.array_equal(oracle.e4m3_code(grid[keep]), codes[keep])


def test_rounding_is_nearest_ties_to_even_with_saturation():
    grid, codes = _all_finite_e4m3()
    pos = np.sort(np.unique(np.abs(grid)))
    mids = (pos[1:] + pos[:-1]) / 2                     # exact ties
    x = np.concatenate([RNG.standard_normal(300) * 40, RNG.standard_normal(200) * 0.01, mids, -mids,
                        [500.0, -1e6, 448.0001, 2.0 ** -10, 3 * 2.0 ** -10]])
    assert np.array_equal(oracle.e4m3_round(x), _brute_nearest(x, grid, codes))
    assert oracle.e4m3_round(np.array([0.1]))[0] == 13 / 128
    assert oracle.e4m3_round(np.array([1e9, -1e9])).tolist() == [448.0, -448.0]


def test_quantize_rows_closed_forms():
    a = np.array([[1.0, -3.5, 0.25, 2.0], [0.0, 0.0, 0.0, 0.0], [-7.0, 1.0, 6.0, 0.5]], dtype=np.float32)
    q, s = oracle.quantize_rows(a)
    assert s.dtype == np.float32
    assert s[0] == np.float32(3.5) / np.float32(448) and s[1] == 1.0
    assert q[0, 1] == -448.0 and q[2, 0] == -448.0          # the row maximum maps to the format maximum
    assert np.all(q[1] == 0)
    assert np.all(np.abs(q) <= 448)
    # dequantised error per element: at most half a quantum of its binade (relative 2^-4), or
    # half the subnormal quantum for tiny values
    deq = q * s[:, None].astype(np.float64)
    err = np.abs(deq - a)
    assert np.all(err <= np.maximum(np.abs(a) * 2.0 ** -4, 2.0 ** -10 * s[:, None]) * 1.0001)


def test_round_bf16_bit_level():
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: even -> 1; 1 + 3 * 2^-8 -> 1 + 2^-6 (even)
    v = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -7, -2.5])
    assert oracle.round_bf16(v).tolist() == [1.0, 1.0 + 2.0 ** -6, 1.0 + 2.0 ** -7, -2.5]


def _grid_expert(H=8, I=4, seed=1):
    """Inputs and weights on the e4m3 grid whose row maxima make the scales powers of two."""
    rng = np.random.default_rng(seed)
    grid, _ = _all_finite_e4m3()
    small = grid[(np.abs(grid) <= 2) & (np.abs(grid) >= 2 ** -3)]
    def mat(n, m):
        a = rng.choice(small, size=(n, m))
        a[:, 0] = 448.0
        return a
    # row maxima 448 * 2^-15: the scales are exactly 2^-15
    return mat(3, H), (mat(I, H) * 2.0 ** -15, mat(I, H) * 2.0 ** -15, mat(H, I) * 2.0 ** -15)


def test_fp8_expert_equals_fp64_expert_when_quantisation_is_exact():
    # x rows and weight rows on the e4m3 grid with row maximum 448 * 2^-k: the scales are powers
    # of two, every code is exact, so gate and up equal the fp64 products; h is then rounded to
    # bf16 and requantised, so the output is checked against that same rounding of the fp64 h
    X, (Wg, Wu, Wd) = _grid_expert()
    qx, sx = oracle.quantize_rows(X)
    assert np.array_equal(qx * sx[:, None], X)
    G, U = X @ Wg.T, X @ Wu.T
    Hb = oracle.round_bf16(oracle.silu(G) * U)
    qh, sh = oracle.quantize_rows(Hb)
    expect = (qh * sh[:, None].astype(np.float64)) @ Wd.T
    assert np.allclose(oracle.swiglu_ffn_fp8(X, Wg, Wu, Wd), expect, rtol=1e-13, atol=1e-300)


def test_fp8_layer_close_to_fp64_layer():
    rng = np.random.default_rng(5)
    T, H, E, k, I = 16, 32, 6, 2, 16
    x = rng.standard_normal((T, H))
    wr = 0.2 * rng.standard_normal((E, H))
    experts = [tuple(0.2 * rng.standard_normal(s) for s in ((I, H), (I, H), (H, I))) for _ in range(E + 1)]
    r = oracle.route(x, wr, np.zeros(E), k, 3.0)
    a = oracle.moe_sparse(x, r, lambda e: experts[e], E)
    b = oracle.moe_sparse_fp8(x, r, lambda e: experts[e], E)
    rel = np.linalg.norm(b - a) / np.linalg.norm(a)
    assert 1e-3 < rel < 0.1, rel        # quantisation error: present, and of the e4m3 size


# ------------------------------------------------------------------ planted mistakes
def test_pins_catch_ties_away_from_zero(monkeypatch):
    def bad(a):
        a = np.asarray(a, dtype=np.float64)
        mag = np.abs(a)
        with np.errstate(divide="ignore"):
            e = np.maximum(np.floor(np.log2(np.where(mag > 0, mag, 1.0))), -6.0)
        q = np.exp2(e - 3.0)
        return np.copysign(np.minimum(np.floor(mag / q + 0.5) * q, 448.0), a)
    monkeypatch.setattr(oracle, "e4m3_round", bad)
    with pytest.raises(AssertionError):
        test_rounding_is_nearest_ties_to_even_with_saturation()


def test_pins_catch_scale_without_the_format_maximum(monkeypatch):
    real = oracle.fp8.quantize_rows

    def bad(a):
        a32 = np.asarray(a, dtype=np.float32)
        amax = np.max(np.abs(a32), axis=-1)
        s = np.where(amax > 0, amax, np.float32(1.0)).astype(np.float32)
        return oracle.e4m3_round((a32 / s[..., None]).astype(np.float32)), s
    monkeypatch.setattr(oracle, "quantize_rows", bad)
    with pytest.raises(AssertionError):
        test_quantize_rows_closed_forms()
    assert real is not bad


def test_fp32_rounding_path_equals_the_arithmetic_one():
    """e4m3_round of an fp32 array rounds on the bit pattern; it must give what the arithmetic
    path gives for the same values in fp64: across the binades, the subnormals, saturation and
    every midpoint between neighbouring e4m3 values (ties to even)."""
    rng = np.random.default_rng(17)
    a = (rng.standard_normal(200_000) * np.exp2(rng.integers(-14, 10, 200_000))).astype(np.float32)
    grid = np.unique(np.abs(oracle.e4m3_decode(np.arange(256, dtype=np.uint8))))
    grid = grid[np.isfinite(grid)]
    mids = ((grid[:-1] + grid[1:]) / 2).astype(np.float32)
    special = np.array([0.0, -0.0, 448, 449, 464, 480, 1e6, -1e6, 2.0 ** -10, -(2.0 ** -10)], dtype=np.float32)
    for v in (a, mids, -mids, special):
        fast = oracle.e4m3_round(v)
        slow = oracle.e4m3_round(v.astype(np.float64))
        assert np.array_equal(fast, slow) and np.array_equal(np.signbit(fast), np.signbit(slow))
