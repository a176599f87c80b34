"""smoe_route_noalloc, the router for callers that cannot allocate device memory (a plugin handed
only its input and output buffers, or a serving path where cudaMalloc is forbidden after
start-up): through the C-ABI, its results must equal smoe_route's, which uses a caller-provided
workspace, on two calls in a row with different batches. The second call also checks that
nothing left in the shared static scratch by the first call leaks into the second.

This file is collected last on purpose, so a run that stops at the first failure has already
run every other test; it also passes when run alone in a fresh process.
"""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import sparse_moe_layer_smoe_b200 as smoe  # noqa: E402


def _route_both(w, x, wr, bias):
    cfg = smoe.config(w.H, w.E, w.k, w.I, w.Is, w.route_scale)
    T = x.shape[0]
    out = {}
    for kind in ("workspace", "noalloc"):
        idx = torch.full((T, w.k), -1, dtype=torch.int32, device="cuda")
        wt = torch.full((T, w.k), float("nan"), dtype=torch.float32, device="cuda")
        logits = torch.full((T, w.E), float("nan"), dtype=torch.float32, device="cuda")
        if kind == "workspace":
            ws = smoe.workspace(cfg, T, forward=False)
            smoe.smoe_route(cfg, x, T, wr, bias, idx, wt, logits, ws)
        else:
            smoe.smoe_route_noalloc(cfg, x, T, wr, bias, idx, wt, logits)
        torch.cuda.synchronize()
        out[kind] = (idx.cpu().numpy(), wt.cpu().numpy(), logits.cpu().numpy())
    return out


def test_route_noalloc_matches_route_on_two_calls_in_a_row():
    w = synth.WORKLOADS["decode"]
    wr, _ = synth.dev_router(w)
    batches = [("decode", synth.WORKLOADS["decode"]), ("mtp", synth.WORKLOADS["mtp"])]
    for name, wb in batches:
        x = synth.dev_x(wb)
        bias = torch.from_numpy(synth.host_bias(wb)).cuda()
        r = _route_both(wb, x, wr, bias)
        (i0, w0, l0), (i1, w1, l1) = r["workspace"], r["noalloc"]
        assert np.array_equal(i0, i1), name
        # same kernels, same reduction order: the tolerance the route tests use (rel 1e-5) holds
        # with room to spare; the results are in fact identical
        assert np.allclose(w1, w0, rtol=1e-5, atol=0), name
        assert np.allclose(l1, l0, rtol=1e-5, atol=1e-6), name
        assert np.all(np.isfinite(w1)) and np.all(np.isfinite(l1))
        assert np.allclose(w1.sum(axis=1), wb.route_scale, rtol=1e-6)


def test_route_noalloc_rejects_sizes_beyond_its_scratch():
    w = synth.WORKLOADS["prefill"]
    cfg = smoe.config(w.H, w.E, w.k, w.I, w.Is, w.route_scale)
    T = 16384   # needs 16384 x 288 x 4 bytes = 18.9 MB of partial logits > 16 MiB
    with pytest.raises(smoe.SmoeError) as ei:
        smoe.smoe_route_noalloc(cfg, 256, T, 256, 256, 256, 256, None)
    assert ei.value.status == smoe.SMOE_ERR_WORKSPACE
