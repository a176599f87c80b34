"""GPU parity of smoe_forward_diag (the layer's monitoring outputs) against the fp64 oracle.

* counts: exact, for the GPU's own selection (a near-tie token may pick another valid set);
* per-expert mean / max expert-output norms: within 5e-3 relative of fp64 ||F_e(x_t)|| (the GPU
  takes the norm of its bf16 output rows); every expert for the tiny layer, a sample of experts
  (the busiest and some random ones) at the Step shape;
* token confidence: within 1e-5 relative (fp32 sigmoid);
* summary: the oracle's summarise() applied to the GPU's own per-expert arrays (checks the
  aggregation kernel), and for the tiny layer the oracle's summary outright;
* the layer output is bit-identical to smoe_forward's, and the whole call is deterministic.
"""
import numpy as np
import pytest

import oracle
import synth
from layer_fixtures import HostExperts, cfg_of, device_inputs, host_route, host_x64, selection_ok

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import sparse_moe_layer_smoe_b200 as smoe  # noqa: E402

RNG = np.random.default_rng(77)


def _run(name, x=None, bias=None, T=None):
    w, x0, wr, bias0, packed = device_inputs(name)
    x = x0 if x is None else x
    bias = bias0 if bias is None else bias
    T = w.T if T is None else T
    cfg = cfg_of(w)
    ws = smoe.workspace(cfg, T)
    out = torch.empty(T, w.H, dtype=torch.bfloat16, device="cuda")
    diag = smoe.diag_buffers(cfg, T)
    smoe.smoe_forward_diag(cfg, x, T, wr, bias, packed, out, diag, ws)
    assert smoe.smoe_get_device_error(ws) == 0
    ref_out = torch.empty_like(out)
    smoe.smoe_forward(cfg, x, T, wr, bias, packed, ref_out, smoe.workspace(cfg, T))
    idx = torch.empty(T, w.k, dtype=torch.int32, device="cuda")
    wt = torch.empty(T, w.k, dtype=torch.float32, device="cuda")
    smoe.smoe_route(cfg, x, T, wr, bias, idx, wt, None, smoe.workspace(cfg, T, forward=False))
    torch.cuda.synchronize()
    return w, out, ref_out, {k: v.cpu().numpy() for k, v in diag.items()}, idx.cpu().numpy()


def _gpu_route(r: oracle.Route, gi: np.ndarray, k: int) -> oracle.Route:
    """The oracle's route with the GPU's selection (checked valid token by token)."""
    for t in range(gi.shape[0]):
        ok, _ = selection_ok(r, t, tuple(sorted(gi[t].tolist())), k)
        assert ok, f"token {t}"
    idx = gi.astype(np.int64)
    s_sel = np.take_along_axis(r.s, idx, axis=1)
    return oracle.Route(r.logits, r.s, r.bhat, idx, s_sel, r.gap)


def _check(name, w, out, ref_out, d, r, x64, experts, check_experts):
    T, k, E = r.idx.shape[0], w.k, w.E
    assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16)), "diagnostics changed the layer output"
    assert np.array_equal(d["expert_count"], np.bincount(r.idx.reshape(-1), minlength=E))
    conf = np.take_along_axis(r.s, r.idx, axis=1).mean(axis=1)
    assert np.allclose(d["token_confidence"][:T], conf, rtol=1e-5, atol=0)
    # summary: the oracle's aggregation applied to the GPU's per-expert arrays
    s_ref = oracle.summarise(d["expert_count"], d["expert_norm_mean"].astype(np.float64),
                             d["expert_norm_max"].astype(np.float64), d["token_confidence"][:T].astype(np.float64),
                             T, k)
    assert np.allclose(d["summary"], s_ref, rtol=2e-6, atol=0), (d["summary"], s_ref)
    # per-expert norms against fp64 expert outputs
    for e in check_experts:
        rows, slots = np.nonzero(r.idx == e)
        if rows.size == 0:
            assert d["expert_norm_mean"][e] == 0 and d["expert_norm_max"][e] == 0
            continue
        y = oracle.swiglu_ffn(x64[rows], *experts(int(e)), limit=w.swiglu_limit)
        n = np.sqrt(np.sum(y * y, axis=1))
        assert np.isclose(d["expert_norm_mean"][e], n.mean(), rtol=5e-3), (e, d["expert_norm_mean"][e], n.mean())
        assert np.isclose(d["expert_norm_max"][e], n.max(), rtol=5e-3), (e, d["expert_norm_max"][e], n.max())


def test_diag_tiny_against_full_oracle():
    w, out, ref_out, d, gi = _run("tiny")
    r = _gpu_route(host_route("tiny"), gi, w.k)
    x64 = host_x64("tiny")
    experts = HostExperts(w, cap=64)
    _check("tiny", w, out, ref_out, d, r, x64, experts, range(w.E))
    full = oracle.diagnostics(x64, r, experts, w.E, limit=w.swiglu_limit)
    assert np.allclose(d["summary"], full.summary, rtol=5e-3, atol=0), (d["summary"], full.summary)
    assert np.allclose(d["expert_norm_mean"], full.expert_norm_mean, rtol=5e-3, atol=0)


def test_diag_decode_sampled_experts():
    w, out, ref_out, d, gi = _run("decode")
    r = _gpu_route(host_route("decode"), gi, w.k)
    counts = np.bincount(r.idx.reshape(-1), minlength=w.E)
    busiest = np.argsort(-counts, kind="stable")[:4].tolist()
    sample = sorted(set(busiest) | set(RNG.choice(w.E, 6, replace=False).tolist()))
    _check("decode", w, out, ref_out, d, r, host_x64("decode"), HostExperts(w, cap=4), sample)


def test_diag_skewed_rows_with_dead_experts_and_determinism():
    """The first 96 tokens of the skewed batch with its Zipf bias: 16 dead experts and many
    experts without tokens; zero counts give zero norms and drop out of the ratios."""
    w = synth.WORKLOADS["skewed"]
    T = 96
    xh = synth.host_x_rows(w, np.arange(T))
    x = torch.from_numpy(xh.view(np.int16)).cuda().view(torch.bfloat16)
    bias = torch.from_numpy(synth.host_bias(w)).cuda()
    w_, out, ref_out, d, gi = _run("skewed", x=x, bias=bias, T=T)
    x64 = oracle.bf16_to_f64(xh)
    r0 = oracle.route(x64, oracle.f32_to_f64(synth.host_w_router(w)), synth.host_bias(w).astype(np.float64), w.k,
                      w.route_scale)
    r = _gpu_route(r0, gi, w.k)
    counts = np.bincount(r.idx.reshape(-1), minlength=w.E)
    assert (counts == 0).sum() >= 16
    dead = np.nonzero(counts == 0)[0][:3].tolist()
    busiest = np.argsort(-counts, kind="stable")[:3].tolist()
    _check("skewed[:96]", w, out, ref_out, d, r, x64, HostExperts(w, cap=4), dead + busiest)
    assert d["summary"][smoe.SMOE_DIAG_ACTIVE_EXPERTS] == (counts > 0).sum()
    # determinism: a second call gives the same bits everywhere
    _, out2, _, d2, _ = _run("skewed", x=x, bias=bias, T=T)
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
    for key in d:
        assert np.array_equal(d[key], d2[key]), key
