"""The gate/up epilogue's arithmetic against fp64: SiLU(g) * u as the GEMM epilogue computes it
from its fp32 accumulators (fast exponential and reciprocal on the special-function unit).
SiLU(z) = z / (1 + e^-z) is the expert activation (Step 3.5 Flash summary, paperlayer.ai, §B:
SwiGLU gate and up projections).

Bound: relative error <= 2^-18 for |g| <= 16 (the exponential's argument error grows with |g|),
far below the bf16 rounding of h (2^-9) that follows; closed forms SiLU(0) = 0 and
SiLU(ln 3) = 3/4 ln 3; SiLU(g) -> g for large g and -> 0 for g -> -inf.
"""
import math

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import sparse_moe_layer_smoe_b200 as smoe  # noqa: E402


def _run(g, u):
    gd = torch.from_numpy(g).cuda()
    ud = torch.from_numpy(u).cuda()
    out = torch.empty_like(gd)
    smoe.smoe_selftest_swiglu(gd, ud, g.size, out)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def _ref(g, u):
    g64, u64 = g.astype(np.float64), u.astype(np.float64)
    with np.errstate(over="ignore"):
        return g64 / (1.0 + np.exp(-g64)) * u64


def test_swiglu_within_bound():
    rng = np.random.default_rng(11)
    g = np.concatenate([np.linspace(-16, 16, 200001), rng.standard_normal(100000) * 4]).astype(np.float32)
    u = rng.standard_normal(g.size).astype(np.float32) * 3 + 0.5
    out, ref = _run(g, u), _ref(g, u)
    tol = 2.0 ** -18 * np.abs(ref) + 1e-30
    assert np.all(np.abs(out - ref) <= tol), np.max(np.abs(out - ref) / np.maximum(np.abs(ref), 1e-30))


def test_swiglu_extremes_and_closed_forms():
    g = np.array([0.0, -0.0, math.log(3.0), 20.0, 60.0, -20.0, -60.0, -87.0, -100.0, -1e30, 1e30], dtype=np.float32)
    out, ref = _run(g, np.ones_like(g)), _ref(g, np.ones_like(g))
    assert out[0] == 0.0 and out[1] == 0.0                          # SiLU(0) = 0
    assert abs(out[2] - 0.75 * math.log(3.0)) <= 2.0 ** -20         # SiLU(ln 3) = 3/4 ln 3
    assert abs(out[3] - ref[3]) <= 2.0 ** -18 * ref[3] and abs(out[4] - 60.0) <= 2.0 ** -18 * 60.0
    assert np.all(np.abs(out[5:9] - ref[5:9]) <= 2.0 ** -18 * np.abs(ref[5:9]) + 1e-40)
    assert out[9] == 0.0                                            # g -> -inf: SiLU -> 0
    assert abs(out[10] - 1e30) <= 1e24                               # g -> +inf: SiLU -> g
