"""fp64 oracle of the layer with FP8 (e4m3) expert weights and activations.

TEST INFRASTRUCTURE, like the rest of ``oracle/``: only ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU leg may import it; the CUDA library shares no code with it.

Source: the Step 3.5 Flash summary (paperlayer.ai) fits the model into a 128 GB workstation
budget, which implies a low-precision format for the experts, but names none. The format and
the quantiser here are readings, stated once and used on both sides:

1. e4m3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits, subnormals, largest finite
   value 448; rounding to nearest, ties to even; values beyond +-448 saturate to +-448;
2. symmetric scaling per row of a matrix (a row = one output feature of a weight matrix, or one
   token of an activation matrix): s = max|row| / 448 in fp32 (s = 1 for an all-zero row), and
   the code of a value a is e4m3(a / s) with a / s rounded to fp32 first. Both divisions are
   IEEE fp32 on both sides, so the codes are a pure function of the inputs (bit-exact parity);
3. the expert: x_t and the gate / up / down weight rows are quantised this way; gate and up are
   sums of code products scaled by s_w s_x; SiLU(g) * up (with the SwiGLU clamp when set) is
   rounded to bf16 (as the bf16 layer does) and then quantised per token for the down product,
   which is scaled by s_w s_h. The router, the combine weights and the shared add stay as in the
   bf16 layer.

Every arithmetic step other than the quantisation decisions is fp64 with no rounding.
"""
from __future__ import annotations

import numpy as np

from .moe import ExpertFn, Route, silu

E4M3_MAX = 448.0


def e4m3_round(a: np.ndarray) -> np.ndarray:
    """Nearest e4m3 value (ties to even mantissa), saturating at +-448; exact in fp64.

    fp32 input takes an equivalent path on the bit pattern (the quantiser's inputs are fp32);
    anything else the arithmetic one below."""
    if isinstance(a, np.ndarray) and a.dtype == np.float32:
        return _e4m3_round_f32(a)
    a = np.asarray(a, dtype=np.float64)
    mag = np.abs(a)
    # binade exponent, clamped at the subnormal range (the quantum there is 2^-9)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(mag > 0, mag, 1.0)))
    e = np.maximum(e, -6.0)
    q = np.exp2(e - 3.0)
    r = np.rint(mag / q) * q          # mag / q is exact (q a power of two); rint: half to even
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, a)


def _e4m3_round_f32(a: np.ndarray) -> np.ndarray:
    """e4m3_round for fp32 values. In the normal e4m3 binades (|a| >= 2^-6) keeping 3 of fp32's
    23 mantissa bits with round-to-nearest-even is integer arithmetic on the bit pattern: add
    0x7FFFF plus the lowest kept bit, then clear the 20 dropped bits (a carry moves into the
    exponent, as rounding up to the next binade should). Below 2^-6 the e4m3 quantum is 2^-9:
    |a| * 2^9 is exact and rint rounds half to even. Then saturation at 448."""
    u = a.view(np.uint32)
    mag_u = u & np.uint32(0x7FFFFFFF)
    lsb = (mag_u >> np.uint32(20)) & np.uint32(1)
    rounded = ((mag_u + np.uint32(0x7FFFF) + lsb) & np.uint32(0xFFF00000)).view(np.float32).astype(np.float64)
    mag = np.abs(a.astype(np.float64))
    sub = mag < 2.0 ** -6
    r = np.where(sub, np.rint(mag * 2.0 ** 9) * 2.0 ** -9, rounded)
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, a.astype(np.float64))


def e4m3_code(v: np.ndarray) -> np.ndarray:
    """uint8 code of values already on the e4m3 grid (sign << 7 | exponent << 3 | mantissa)."""
    v = np.asarray(v, dtype=np.float64)
    sign = (np.signbit(v)).astype(np.uint8) << 7
    mag = np.abs(v)
    out = np.zeros(v.shape, dtype=np.uint8)
    sub = mag < 2.0 ** -6
    out[sub] = np.rint(mag[sub] / 2.0 ** -9).astype(np.uint8)              # exponent field 0
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(sub, 1.0, mag)))
    m = np.rint((np.where(sub, 1.0, mag) / np.exp2(e) - 1.0) * 8.0)
    norm = ~sub
    out[norm] = (((e[norm] + 7).astype(np.uint8) << 3) | m[norm].astype(np.uint8))
    return out | sign


def e4m3_decode(code: np.ndarray) -> np.ndarray:
    """Value of uint8 e4m3 codes (NaN for the two NaN codes)."""
    c = np.asarray(code, dtype=np.uint8).astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    ex = (c >> 3) & 0xF
    man = c & 0x7
    val = np.where(ex == 0, man * 2.0 ** -9, (1.0 + man / 8.0) * np.exp2(ex - 7.0))
    val = np.where((ex == 0xF) & (man == 0x7), np.nan, val)
    return s * val


def quantize_rows(a: np.ndarray):
    """Per-row symmetric e4m3 quantisation (reading 2): (values on the e4m3 grid as fp64, fp32 scales)."""
    a32 = np.asarray(a, dtype=np.float32)
    amax = np.max(np.abs(a32), axis=-1)
    s = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    scaled = (a32 / s[..., None]).astype(np.float32)
    return e4m3_round(scaled), s   # fp32 in: the bit-pattern path


def round_bf16(a: np.ndarray) -> np.ndarray:
    """fp64 -> nearest bf16 (ties to even), via fp32 (an fp64 value rounds to fp32 first)."""
    f = np.asarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


class QuantExpert(tuple):
    """An expert's weights already quantised per row (reading 2): (qg, sg, qu, su, qd, sd), the
    values on the e4m3 grid as fp64 and the fp32 row scales. An ExpertFn may return one of these
    instead of the bf16 weights, so that a caller can quantise each expert once."""


def quantize_expert(Wg: np.ndarray, Wu: np.ndarray, Wd: np.ndarray) -> QuantExpert:
    qg, sg = quantize_rows(Wg)
    qu, su = quantize_rows(Wu)
    qd, sd = quantize_rows(Wd)
    return QuantExpert((qg, sg, qu, su, qd, sd))


def swiglu_ffn_fp8(X: np.ndarray, Wg, Wu=None, Wd=None, limit: float = 0.0) -> np.ndarray:
    """F_q(X) for rows X [n, H] with fp64 weights (bf16 values), or with one QuantExpert in place
    of the three weights: reading 3."""
    qg, sg, qu, su, qd, sd = Wg if isinstance(Wg, QuantExpert) else quantize_expert(Wg, Wu, Wd)
    qx, sx = quantize_rows(X)
    sx64 = sx.astype(np.float64)[:, None]
    G = (qx @ qg.T) * sx64 * sg.astype(np.float64)[None, :]
    U = (qx @ qu.T) * sx64 * su.astype(np.float64)[None, :]
    if limit > 0:
        G = np.minimum(G, limit)
        U = np.clip(U, -limit, limit)
    Hb = round_bf16(silu(G) * U)
    qh, sh = quantize_rows(Hb)
    return (qh @ qd.T) * sh.astype(np.float64)[:, None] * sd.astype(np.float64)[None, :]


def moe_sparse_fp8(x: np.ndarray, r: Route, expert: ExpertFn, E: int, limit: float = 0.0,
                   limit_shared: float = 0.0) -> np.ndarray:
    """out[t] = F_q,shared(x_t) + sum_j w[t, j] F_q,idx[t, j](x_t) over the selected experts."""
    def weights(e):
        w = expert(e)
        return (w,) if isinstance(w, QuantExpert) else tuple(w)
    out = swiglu_ffn_fp8(x, *weights(E), limit=limit_shared)
    for e in np.unique(r.idx):
        rows, slots = np.nonzero(r.idx == e)
        out[rows] += r.w[rows, slots][:, None] * swiglu_ffn_fp8(x[rows], *weights(int(e)), limit=limit)
    return out
