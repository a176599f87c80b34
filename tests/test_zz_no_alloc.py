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

import oracle
import synth
from layer_fixtures import selection_ok

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
    # both batches below the tensor-core router's size, so both entry points run the same kernels
    batches = [("decode", synth.WORKLOADS["decode"], 64), ("mtp rows 0-299", synth.WORKLOADS["mtp"], 300)]
    for name, wb, rows in batches:
        x = synth.dev_x(wb)[:rows].contiguous()
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


def test_route_noalloc_mid_batch_matches_the_oracle():
    """At 600 tokens smoe_route runs on the tensor cores, the allocation-free router on the CUDA
    cores (64-token x 96-expert tiles): checked against the fp64 oracle directly."""
    w = synth.WORKLOADS["prefill"]
    T = 600
    cfg = smoe.config(w.H, w.E, w.k, w.I, w.Is, w.route_scale)
    xh = synth.host_x_rows(w, np.arange(T))
    x = torch.from_numpy(xh.view(np.int16)).cuda().view(torch.bfloat16)
    wr, _ = synth.dev_router(w)
    bias_h = synth.host_bias(w)
    idx = torch.empty(T, w.k, dtype=torch.int32, device="cuda")
    wt = torch.empty(T, w.k, dtype=torch.float32, device="cuda")
    smoe.smoe_route_noalloc(cfg, x, T, wr, torch.from_numpy(bias_h).cuda(), idx, wt, None)
    gi, gw = idx.cpu().numpy(), wt.cpu().numpy().astype(np.float64)
    r = oracle.route(oracle.bf16_to_f64(xh), oracle.f32_to_f64(synth.host_w_router(w)), bias_h.astype(np.float64),
                     w.k, w.route_scale)
    for t in range(T):
        ok, _ = selection_ok(r, t, tuple(sorted(gi[t].tolist())), w.k)
        assert ok, f"token {t}"
        if not r.near_tie[t]:
            ref_w = dict(zip(r.idx[t].tolist(), r.w[t].tolist()))
            assert np.allclose(gw[t], [ref_w[e] for e in gi[t].tolist()], rtol=1e-5, atol=0), f"token {t}"


def _sentinel_outputs(T, w):
    idx = torch.full((T, w.k), -7, dtype=torch.int32, device="cuda")
    wt = torch.full((T, w.k), -3.5, dtype=torch.float32, device="cuda")
    return idx, wt


def test_route_noalloc_limit_is_the_documented_one():
    """At E = 288 large batches run with a K split of 1, so the static 16 MiB array holds the
    partial logits of floor(16 MiB / (288 x 4)) = 14,563 tokens. One token more is refused with
    SMOE_ERR_WORKSPACE before any launch: the real output buffers keep their sentinels."""
    w = synth.WORKLOADS["prefill"]
    cfg = smoe.config(w.H, w.E, w.k, w.I, w.Is, w.route_scale)
    t_max = smoe.SMOE_NOALLOC_SCRATCH_BYTES // (w.E * 4)
    assert t_max == 14563
    wr, bias = synth.dev_router(w)
    x = torch.empty(t_max + 1, w.H, dtype=torch.bfloat16, device="cuda")
    synth.dev_fill(x, 3, synth.TID_X, 1.0)
    # one token beyond the limit: refused, nothing written
    idx, wt = _sentinel_outputs(t_max + 1, w)
    with pytest.raises(smoe.SmoeError) as ei:
        smoe.smoe_route_noalloc(cfg, x, t_max + 1, wr, bias, idx, wt, None)
    assert ei.value.status == smoe.SMOE_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((idx == -7).all()) and bool((wt == -3.5).all())
    # at the limit: accepted, and every token routed to k distinct experts with weights summing to 3
    xm = x[:t_max]
    idx, wt = _sentinel_outputs(t_max, w)
    smoe.smoe_route_noalloc(cfg, xm, t_max, wr, bias, idx, wt, None)
    torch.cuda.synchronize()
    gi = idx.cpu().numpy()
    assert gi.min() >= 0 and gi.max() < w.E
    assert np.all(np.sort(gi, axis=1)[:, 1:] != np.sort(gi, axis=1)[:, :-1])
    assert torch.allclose(wt.sum(dim=1), torch.full((t_max,), w.route_scale, device="cuda"), rtol=1e-6)
    # and the same selections as smoe_route on a slice of it (sets compared; order and near ties
    # are covered by the oracle tests above)
    ref_idx, ref_wt = _sentinel_outputs(1024, w)
    ws = smoe.workspace(cfg, 1024, forward=False)
    smoe.smoe_route(cfg, xm[:1024].contiguous(), 1024, wr, bias, ref_idx, ref_wt, None, ws)
    torch.cuda.synchronize()
    same = (np.sort(gi[:1024], axis=1) == np.sort(ref_idx.cpu().numpy(), axis=1)).all(axis=1)
    assert same.mean() > 0.99


def test_route_noalloc_on_every_visible_device():
    """The array's address is looked up in the current context on every call, so each device
    (made current by torch) uses its own copy: results equal smoe_route's on each of them."""
    w = synth.WORKLOADS["decode"]
    cfg = smoe.config(w.H, w.E, w.k, w.I, w.Is, w.route_scale)
    prev = torch.cuda.current_device()
    try:
        for d in range(torch.cuda.device_count()):
            torch.cuda.set_device(d)
            wr, bias = synth.dev_router(w, device=f"cuda:{d}")
            x = synth.dev_x(w, device=f"cuda:{d}")
            r = _route_both(w, x, wr, bias)
            assert np.array_equal(r["workspace"][0], r["noalloc"][0]), f"device {d}"
            assert np.array_equal(r["workspace"][1], r["noalloc"][1]), f"device {d}"
    finally:
        torch.cuda.set_device(prev)
