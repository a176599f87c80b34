"""GPU parity: every call of libstepmoe (through the C-ABI) against the fp64 oracle on the same
seeded inputs, on all five workloads, at their full sizes.

* generator: device fill == host fill, bit for bit (both sides' inputs are the same values);
* route: the selected set bit-exact except near ties (valid-band check); the order within it
  descending by oracle biased score up to inner ties closer than 1e-5; weights rel 1e-5,
  fp32 logits within an fp32 accumulation bound;
* permute: counts, offsets, perm_row, row_token and x_perm bit-exact;
* expert_ffn: fed the oracle's permutation, outputs vs fp64 SwiGLU experts (all rows for the
  tiny layer; at the Step shape rows from every (group, token tile), both halves of each tile
  and every trimmed tail tile, the shared expert's tiles included);
* combine: fed seeded bf16 rows and the oracle's weights, vs the fp64 formula within 1 bf16 ulp;
* forward (the launch configuration bench.py times): the whole layer vs the oracle, dense-masked
  for tiny and decode, sparse on >= 256 tokens spread over the batch (plus near-tie and spike
  rows) otherwise; and a
  degenerate routing collapse (every token to the same 8 experts) on both GEMM kernels.
"""
import numpy as np
import pytest

import oracle
import synth
from layer_fixtures import (ALL_WORKLOADS, HostExperts, assert_close, bf16_tensor_to_f64, cfg_of, device_inputs,
                            host_route, host_x64, limit_of, selection_ok, stratified_tokens)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import sparse_moe_layer_smoe_b200 as smoe  # noqa: E402

RNG = np.random.default_rng(2024)


def _ws(cfg, T, forward=False):
    return smoe.workspace(cfg, T, forward=forward)


# ------------------------------------------------------------------------------ generator
def test_device_generator_matches_host():
    w = synth.WORKLOADS["mtp"]
    x = synth.dev_x(w)
    xh = synth.host_x(w)
    assert np.array_equal(x.cpu().view(torch.int16).numpy().view(np.uint16), xh)
    wr, _ = synth.dev_router(w)
    assert np.array_equal(wr.cpu().numpy().view(np.uint32), synth.host_w_router(w).view(np.uint32))
    t = torch.empty(3 * 1280 * 4096, dtype=torch.bfloat16, device="cuda")
    synth.dev_fill(t, 0, synth.TID_WD, 0.02, index_base=77 * 1280 * 4096)
    h = synth.host_bf16(t.numel(), 0, synth.TID_WD, 0.02, index_base=77 * 1280 * 4096)
    assert np.array_equal(t.cpu().view(torch.int16).numpy().view(np.uint16), h)


# ------------------------------------------------------------------------------ route
@pytest.mark.parametrize("name", ALL_WORKLOADS)
def test_route_parity(name):
    w, x, wr, bias, _ = device_inputs(name)
    cfg = cfg_of(w)
    T = w.T
    idx = torch.empty(T, w.k, dtype=torch.int32, device="cuda")
    wt = torch.empty(T, w.k, dtype=torch.float32, device="cuda")
    logits = torch.empty(T, w.E, dtype=torch.float32, device="cuda")
    ws = _ws(cfg, T)
    smoe.smoe_route(cfg, x, T, wr, bias, idx, wt, logits, ws)
    assert smoe.smoe_get_device_error(ws) == 0
    r = host_route(name)
    gi, gw, gl = idx.cpu().numpy(), wt.cpu().numpy().astype(np.float64), logits.cpu().numpy().astype(np.float64)

    # fp32 logits: error of an fp32 dot product of length H, scaled by the row's magnitude
    scale = np.abs(host_x64(name)).max(axis=1, keepdims=True) * 0.1 + 1.0
    assert np.all(np.abs(gl - r.logits) <= 2e-4 * scale), np.abs(gl - r.logits).max()

    near = swapped = 0
    for t in range(T):
        gset = tuple(sorted(gi[t].tolist()))
        assert len(set(gset)) == w.k and min(gset) >= 0 and max(gset) < w.E
        ok, ref_set = selection_ok(r, t, gset, w.k)
        assert ok, f"token {t}: GPU selection {gset} vs oracle {tuple(sorted(r.idx[t].tolist()))}"
        if r.near_tie[t]:
            near += 1
        # order: descending oracle biased score, up to inner ties closer than the tie tolerance
        b = r.bhat[t, gi[t]]
        assert np.all(b[:-1] >= b[1:] - oracle.NEAR_TIE_EPS), f"token {t}: order {gi[t]} vs {r.idx[t]}"
        swapped += int(gset == tuple(sorted(r.idx[t].tolist())) and not np.array_equal(gi[t], r.idx[t]))
        if not r.near_tie[t]:
            # weights matched by expert id: the oracle's weight of each selected expert
            ref_w = dict(zip(r.idx[t].tolist(), r.w[t].tolist()))
            assert np.allclose(gw[t], [ref_w[e] for e in gi[t].tolist()], rtol=1e-5, atol=0), f"token {t}: weights"
        else:
            s_sel = r.s[t, gi[t]]
            assert np.allclose(gw[t], oracle.normalise(s_sel, w.route_scale), rtol=1e-5, atol=0)
    assert np.allclose(gw.sum(axis=1), w.route_scale, rtol=1e-6)
    print(f"{name}: {near} near-tie tokens of {T}; {swapped} tokens with the oracle's set in another order "
          f"(every swap within the 1e-5 band)")


@pytest.mark.parametrize("T", [37, 700, 2100])   # the small-batch, mid-batch and tensor-core router plans
def test_route_exact_ties_follow_the_tie_rule(T):
    """Rows of zeros give every expert the logit 0 and the score 1/2 exactly, so biases drawn
    from {-1/4, 0, 1/4} tie the biased scores exactly within each bias class: the selection is
    then fixed by the tie rule alone (larger logit, all equal here, then smaller index) and must
    match bit for bit, with every weight 3/8. The other rows carry Step-shape inputs."""
    w = synth.WORKLOADS["decode"]
    cfg = cfg_of(w)
    E, k = w.E, w.k
    wr = device_inputs("decode")[2]
    xb = synth.host_bf16(T * w.H, 5, synth.TID_X, 1.0).reshape(T, w.H)
    zero = np.arange(T) % 3 == 0
    xb[zero] = 0
    bias = np.random.default_rng(T).choice(np.array([-0.25, 0.0, 0.25], dtype=np.float32), size=E)
    x = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    wt = torch.empty(T, k, dtype=torch.float32, device="cuda")
    ws = _ws(cfg, T)
    smoe.smoe_route(cfg, x, T, wr, torch.from_numpy(bias).cuda(), idx, wt, None, ws)
    gi, gw = idx.cpu().numpy(), wt.cpu().numpy()
    r = oracle.route(oracle.bf16_to_f64(xb), oracle.f32_to_f64(synth.host_w_router(w)), bias.astype(np.float64), k,
                     w.route_scale)
    expect = np.lexsort((np.arange(E), -bias.astype(np.float64)))[:k]
    for t in np.nonzero(zero)[0]:
        assert np.array_equal(r.idx[t], expect)
        assert np.array_equal(gi[t], expect), f"token {t}: {gi[t]} vs {expect}"
        assert np.all(gw[t] == np.float32(w.route_scale / k))
    for t in np.nonzero(~zero)[0]:
        ok, _ = selection_ok(r, t, tuple(sorted(gi[t].tolist())), k)
        assert ok, f"token {t}"


# ------------------------------------------------------------------------------ permute
@pytest.mark.parametrize("name", ALL_WORKLOADS)
def test_permute_parity(name):
    w, x, _, _, _ = device_inputs(name)
    cfg = cfg_of(w)
    T, k, E = w.T, w.k, w.E
    r = host_route(name)
    idx = torch.from_numpy(r.idx).cuda()
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm_row = torch.empty(T * k, dtype=torch.int32, device="cuda")
    row_token = torch.empty(T * k, dtype=torch.int32, device="cuda")
    x_perm = torch.empty(T * k, w.H, dtype=torch.bfloat16, device="cuda")
    ws = _ws(cfg, T)
    smoe.smoe_permute(cfg, idx, T, x, counts, offsets, perm_row, row_token, x_perm, ws)
    assert smoe.smoe_get_device_error(ws) == 0
    c, o, p, rt = oracle.permute(r.idx, E)
    assert np.array_equal(counts.cpu().numpy(), c)
    assert np.array_equal(offsets.cpu().numpy(), o)
    assert np.array_equal(perm_row.cpu().numpy(), p)
    assert np.array_equal(row_token.cpu().numpy(), rt)
    xh = synth.host_x(w)
    assert np.array_equal(x_perm.cpu().view(torch.int16).numpy().view(np.uint16), xh[rt])


# ------------------------------------------------------------------------------ expert FFN
def _token_tile_rows(offsets, T, k, rng):
    """Rows of y that reach every (group, token tile) of the expert GEMMs: in each tile its first
    and last rows, the first row of its second half and one random row of each half (a CTA pair
    holds one half of a tile in each CTA), so every trimmed tail tile and the shared expert's
    tiles are checked too. The tiling restates the kernels' documented rule: the launch's largest
    tile is the smallest power of two >= 1.25 x the mean rows per routed expert (16..256), and a
    group of r rows uses the smallest power of two >= r, clamped to [16, that largest tile]."""
    E = len(offsets) - 1
    nt_max = 16
    while nt_max < 256 and nt_max < 1.25 * T * k / E:
        nt_max *= 2
    groups = [(int(offsets[e]), int(offsets[e + 1])) for e in range(E)] + [(T * k, T * k + T)]
    rows = set()
    tiles = 0
    for a, b in groups:
        if b == a:
            continue
        nt = 16
        while nt < b - a and nt < nt_max:
            nt *= 2
        for s in range(a, b, nt):
            end, half = min(s + nt, b), s + nt // 2
            rows |= {s, end - 1, int(rng.integers(s, min(half, end)))}
            if half < end:
                rows |= {half, int(rng.integers(half, end))}
            tiles += 1
    return sorted(rows), tiles


@pytest.mark.parametrize("mode", ["gather", "x_perm"])
@pytest.mark.parametrize("name", ALL_WORKLOADS + ["mtp_clamp"])
def test_expert_ffn_parity(name, mode):
    """gather: routed rows read from x through row_token inside the GEMM; x_perm: from a
    permuted copy of x built on the host from the oracle's permutation."""
    w, x, _, _, packed = device_inputs(name)
    cfg = cfg_of(w)
    T, k, E = w.T, w.k, w.E
    r = host_route(name)
    _, offsets, _, row_token = oracle.permute(r.idx, E)
    xh = synth.host_x(w)
    x_perm = None
    if mode == "x_perm":
        x_perm = torch.from_numpy(xh[row_token].view(np.int16)).cuda().view(torch.bfloat16)
    y = torch.full((T * k + T, w.H), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = _ws(cfg, T)
    smoe.smoe_expert_ffn(cfg, x, x_perm, torch.from_numpy(row_token).cuda(), torch.from_numpy(offsets).cuda(), T,
                         packed, y, ws)
    assert smoe.smoe_get_device_error(ws) == 0
    gy = bf16_tensor_to_f64(y)
    x64 = host_x64(name)
    experts = HostExperts(w)
    group_of = np.searchsorted(offsets, np.arange(T * k), side="right") - 1
    if name == "tiny":
        rows, tiles = list(range(T * k + T)), None
    else:
        rows, tiles = _token_tile_rows(offsets, T, k, RNG)
    if w.bias == "zipf":   # the dead experts own no rows
        dead = np.nonzero(synth.zipf_ranks(w) > w.E - synth.ZIPF_DEAD)[0]
        assert len(dead) == synth.ZIPF_DEAD and np.all(offsets[dead + 1] == offsets[dead])
    spikes = synth.spike_rows(w)
    if len(spikes):   # rows of the x50 spike tokens: routed ones and their shared rows
        rows = sorted(set(rows) | set(np.nonzero(np.isin(row_token, spikes))[0][:6].tolist())
                      | set((T * k + spikes[:2]).tolist()))
    ref = np.empty((len(rows), w.H))
    by_group = {}
    for i, rr in enumerate(rows):
        g, tok = (E, rr - T * k) if rr >= T * k else (int(group_of[rr]), int(row_token[rr]))
        by_group.setdefault(g, []).append((i, tok))
    clamped = 0.0
    for g, items in by_group.items():
        ii = [a for a, _ in items]
        xs = x64[[b for _, b in items]]
        ref[ii] = oracle.swiglu_ffn(xs, *experts(g), limit=limit_of(w, g))
        if limit_of(w, g) > 0:
            clamped = max(clamped, np.abs(ref[ii] - oracle.swiglu_ffn(xs, *experts(g))).max())
    if w.swiglu_limit > 0:
        assert clamped > 0.0   # the sampled rows exercise the clamp
    assert np.all(np.isfinite(gy[rows]))
    fro, mx = assert_close(gy[rows], ref, f"{name} expert_ffn ({mode})")
    assert torch.isfinite(y.float()).all()   # every row written
    print(f"{name}: expert_ffn ({mode}) rows={len(rows)} token tiles={tiles} rel_fro={fro:.2e} rel_max={mx:.2e}")


# ------------------------------------------------------------------------------ combine
@pytest.mark.parametrize("name", ["tiny", "decode", "mtp"])
def test_combine_parity(name):
    w = synth.WORKLOADS[name]
    cfg = cfg_of(w)
    T, k = w.T, w.k
    r = host_route(name)
    _, _, perm_row, _ = oracle.permute(r.idx, w.E)
    yh = synth.host_bf16((T * k + T) * w.H, 5, 99, 1.0).reshape(T * k + T, w.H)
    wt = r.w.astype(np.float32)
    y = torch.from_numpy(yh.view(np.int16)).cuda().view(torch.bfloat16)
    out = torch.empty(T, w.H, dtype=torch.bfloat16, device="cuda")
    ws = _ws(cfg, T)
    smoe.smoe_combine(cfg, y, torch.from_numpy(perm_row).cuda(), torch.from_numpy(wt).cuda(), T, out, ws)
    assert smoe.smoe_get_device_error(ws) == 0
    ref = oracle.combine(oracle.bf16_to_f64(yh), perm_row, wt.astype(np.float64), T, k)
    got = bf16_tensor_to_f64(out)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-6 * (np.abs(oracle.bf16_to_f64(yh)).max() * (k + 1) * 3)
    assert np.all(np.abs(got - ref) <= bound), np.abs(got - ref).max()


# ------------------------------------------------------------------------------ the whole layer
def _forward(name):
    w, x, wr, bias, packed = device_inputs(name)
    cfg = cfg_of(w)
    out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
    ws = _ws(cfg, w.T, forward=True)
    smoe.smoe_forward(cfg, x, w.T, wr, bias, packed, out, ws)
    assert smoe.smoe_get_device_error(ws) == 0
    return w, out, ws


def _layer_rows(name, rows, gi, w, dense):
    """Oracle output rows for the given tokens, and the per-token selection check."""
    r = host_route(name)
    x64 = host_x64(name)
    experts = HostExperts(w, cap=4 if dense else 24)
    sel_rows = []
    for t in rows:
        gset = tuple(sorted(gi[t].tolist()))
        ok, ref_set = selection_ok(r, t, gset, w.k)
        assert ok, f"token {t}: selection {gset}"
        sel_rows.append((t, ref_set))
    sub = oracle.Route(r.logits[rows], r.s[rows], r.bhat[rows], r.idx[rows], r.w[rows], r.gap[rows])
    lim = dict(limit=w.swiglu_limit, limit_shared=w.swiglu_limit_shared)
    if dense:
        ref = oracle.moe_dense_masked(x64[rows], sub, experts, w.E, **lim)
    else:
        ref = oracle.moe_sparse(x64[rows], sub, experts, w.E, **lim)
    for i, (t, ref_set) in enumerate(sel_rows):
        if ref_set != tuple(sorted(r.idx[t].tolist())):
            # near tie resolved to another valid set: the oracle's output for that set
            order = sorted(ref_set, key=lambda e: -r.bhat[t, e])
            ref[i] = oracle.moe_given_selection(x64[t], r.s[t], order, experts, w.E, w.route_scale, **lim)
    return ref


@pytest.mark.parametrize("name", ["tiny", "decode"])
def test_forward_parity_dense_masked(name):
    """Whole layer vs the oracle brute-forcing every expert and masking by the selection."""
    w, out, _ = _forward(name)
    idx = torch.empty(w.T, w.k, dtype=torch.int32, device="cuda")
    wt = torch.empty(w.T, w.k, dtype=torch.float32, device="cuda")
    ws = _ws(cfg_of(w), w.T)
    _, x, wr, bias, _ = device_inputs(name)
    smoe.smoe_route(cfg_of(w), x, w.T, wr, bias, idx, wt, None, ws)
    rows = list(range(w.T))
    ref = _layer_rows(name, rows, idx.cpu().numpy(), w, dense=True)
    fro, mx = assert_close(bf16_tensor_to_f64(out)[rows], ref, f"{name} forward (dense-masked oracle)")
    print(f"{name}: forward rel_fro={fro:.2e} rel_max={mx:.2e}")


@pytest.mark.parametrize("name", ["prefill", "skewed", "mtp", "mtp_clamp"])
def test_forward_parity_sampled(name):
    w, out, _ = _forward(name)
    cfg = cfg_of(w)
    _, x, wr, bias, _ = device_inputs(name)
    idx = torch.empty(w.T, w.k, dtype=torch.int32, device="cuda")
    wt = torch.empty(w.T, w.k, dtype=torch.float32, device="cuda")
    smoe.smoe_route(cfg, x, w.T, wr, bias, idx, wt, None, _ws(cfg, w.T))
    r = host_route(name)
    rows = {0, w.T - 1, *stratified_tokens(w.T, 256, RNG)}
    rows |= set(np.nonzero(r.near_tie)[0][:3].tolist())
    rows |= set(synth.spike_rows(w).tolist())
    rows = sorted(rows)
    ref = _layer_rows(name, rows, idx.cpu().numpy(), w, dense=False)
    got = bf16_tensor_to_f64(out)[rows]
    fro, mx = assert_close(got, ref, f"{name} forward (sampled tokens)")
    # properties at full size: finite output everywhere
    assert torch.isfinite(out.float()).all()
    print(f"{name}: forward rows={len(rows)} rel_fro={fro:.2e} rel_max={mx:.2e} near_ties={int(r.near_tie.sum())}")


@pytest.mark.parametrize("name", ["mtp", "decode"])
def test_forward_is_deterministic_and_matches_per_call_chain(name):
    """smoe_forward twice (same bits), and the same bits as chaining the four calls."""
    w, out1, _ = _forward(name)
    _, out2, _ = _forward(name)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    # chaining the four calls gives the same bits as smoe_forward
    _, x, wr, bias, packed = device_inputs(name)
    cfg = cfg_of(w)
    T, k, E = w.T, w.k, w.E
    ws = _ws(cfg, T)
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    wt = torch.empty(T, k, dtype=torch.float32, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm_row = torch.empty(T * k, dtype=torch.int32, device="cuda")
    row_token = torch.empty(T * k, dtype=torch.int32, device="cuda")
    x_perm = torch.empty(T * k, w.H, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(T * k + T, w.H, dtype=torch.bfloat16, device="cuda")
    out3 = torch.empty(T, w.H, dtype=torch.bfloat16, device="cuda")
    smoe.smoe_route(cfg, x, T, wr, bias, idx, wt, None, ws)
    smoe.smoe_permute(cfg, idx, T, x, counts, offsets, perm_row, row_token, x_perm, ws)
    smoe.smoe_expert_ffn(cfg, x, None, row_token, offsets, T, packed, y, ws)
    smoe.smoe_combine(cfg, y, perm_row, wt, T, out3, ws)
    # the permuted-copy path gives the same bits
    y2 = torch.empty_like(y)
    smoe.smoe_expert_ffn(cfg, x, x_perm, row_token, offsets, T, packed, y2, ws)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    assert smoe.smoe_get_device_error(ws) == 0
    assert torch.equal(out1.view(torch.int16), out3.view(torch.int16))


@pytest.mark.parametrize("T", [1, 3, 17, 255, 257])
def test_forward_ragged_token_counts(T):
    """Ragged T (partial token tiles, one token, across permute block edges) on the tiny layer."""
    w0 = synth.WORKLOADS["tiny"]
    w = synth.Workload("tiny_T", T, w0.H, w0.E, w0.k, w0.I, w0.Is)
    cfg = cfg_of(w)
    _, _, wr, bias, packed = device_inputs("tiny")
    x = synth.dev_x(w)
    out = torch.empty(T, w.H, dtype=torch.bfloat16, device="cuda")
    ws = _ws(cfg, T, forward=True)
    smoe.smoe_forward(cfg, x, T, wr, bias, packed, out, ws)
    assert smoe.smoe_get_device_error(ws) == 0
    x64 = oracle.bf16_to_f64(synth.host_x(w))
    r = oracle.route(x64, oracle.f32_to_f64(synth.host_w_router(w)), synth.host_bias(w).astype(np.float64), w.k,
                     w.route_scale)
    ref = oracle.moe_sparse(x64, r, HostExperts(w), w.E)
    keep = ~r.near_tie   # a near tie may resolve to another valid selection; checked in test_route_parity
    assert_close(bf16_tensor_to_f64(out)[keep], ref[keep], f"tiny T={T}")


@pytest.mark.parametrize("T", [512, 2048])
def test_forward_routing_collapse(T):
    """Degenerate routing (the routing collapse that the loss-free balancing bias is there to
    prevent, pushed to its limit): a bias of +20 on 8 experts sends every token to the same 8, so
    8 groups hold all T*k routed rows, in many token tiles each, and the other 280 are empty
    (single-CTA kernel with 16-row tiles at T=512, CTA pairs with 128-row tiles at T=2048)."""
    w0 = synth.WORKLOADS["mtp"]
    w = synth.Workload("collapse", T, w0.H, w0.E, w0.k, w0.I, w0.Is)
    cfg = cfg_of(w)
    _, _, wr, _, packed = device_inputs("mtp")
    hot = np.array([3, 17, 50, 97, 144, 191, 238, 285])
    bias_h = np.zeros(w.E, dtype=np.float32)
    bias_h[hot] = 20.0
    bias = torch.from_numpy(bias_h).cuda()
    x = synth.dev_x(w)
    out = torch.empty(T, w.H, dtype=torch.bfloat16, device="cuda")
    smoe.smoe_forward(cfg, x, T, wr, bias, packed, out, _ws(cfg, T, forward=True))
    idx = torch.empty(T, w.k, dtype=torch.int32, device="cuda")
    wt = torch.empty(T, w.k, dtype=torch.float32, device="cuda")
    ws = _ws(cfg, T)
    smoe.smoe_route(cfg, x, T, wr, bias, idx, wt, None, ws)
    assert smoe.smoe_get_device_error(ws) == 0
    assert np.array_equal(np.sort(idx.cpu().numpy(), axis=1), np.tile(hot, (T, 1)))
    x64 = oracle.bf16_to_f64(synth.host_x(w))
    r = oracle.route(x64, oracle.f32_to_f64(synth.host_w_router(w)), bias_h.astype(np.float64), w.k, w.route_scale)
    assert np.array_equal(np.sort(r.idx, axis=1), np.tile(hot, (T, 1)))
    rows = sorted({0, T - 1, *RNG.integers(0, T, 6).tolist()})
    sub = oracle.Route(r.logits[rows], r.s[rows], r.bhat[rows], r.idx[rows], r.w[rows], r.gap[rows])
    ref = oracle.moe_sparse(x64[rows], sub, HostExperts(w, cap=9), w.E)
    fro, mx = assert_close(bf16_tensor_to_f64(out)[rows], ref, f"collapse T={T} forward (sampled tokens)")
    assert torch.isfinite(out.float()).all()
    print(f"collapse T={T}: rows={len(rows)} rel_fro={fro:.2e} rel_max={mx:.2e}")


@pytest.mark.parametrize("T", [700, 1024, 1500])
def test_forward_parity_mid_batches(T):
    """Batch sizes between the named workloads, each on another launch plan: T = 700 (tensor-core
    router, 32-token tiles with rows gathered inside the single-CTA GEMM), 1024 (CTA pairs with
    64-token tiles, the one-CTA permutation at its limit) and 1500 (CTA pairs with 64-token tiles,
    the multi-block permutation). The first T tokens of the prefill batch at the Step shape; the
    whole layer against the oracle on 128 tokens spread over the batch."""
    w0 = synth.WORKLOADS["prefill"]
    w = synth.Workload("mid", T, w0.H, w0.E, w0.k, w0.I, w0.Is)
    cfg = cfg_of(w)
    _, _, wr, _, packed = device_inputs("prefill")
    xh = synth.host_x_rows(w0, np.arange(T))
    x = torch.from_numpy(xh.view(np.int16)).cuda().view(torch.bfloat16)
    bias = torch.zeros(w.E, dtype=torch.float32, device="cuda")
    out = torch.empty(T, w.H, dtype=torch.bfloat16, device="cuda")
    ws = _ws(cfg, T, forward=True)
    smoe.smoe_forward(cfg, x, T, wr, bias, packed, out, ws)
    assert smoe.smoe_get_device_error(ws) == 0
    idx = torch.empty(T, w.k, dtype=torch.int32, device="cuda")
    wt = torch.empty(T, w.k, dtype=torch.float32, device="cuda")
    smoe.smoe_route(cfg, x, T, wr, bias, idx, wt, None, _ws(cfg, T))
    gi = idx.cpu().numpy()
    x64 = oracle.bf16_to_f64(xh)
    r = oracle.route(x64, oracle.f32_to_f64(synth.host_w_router(w0)), np.zeros(w.E), w.k, w.route_scale)
    rows = sorted(t for t in stratified_tokens(T, 128, RNG) if not r.near_tie[t])
    for t in rows:
        ok, _ = selection_ok(r, t, tuple(sorted(gi[t].tolist())), w.k)
        assert ok, f"token {t}"
    sub = oracle.Route(r.logits[rows], r.s[rows], r.bhat[rows], r.idx[rows], r.w[rows], r.gap[rows])
    ref = oracle.moe_sparse(x64[rows], sub, HostExperts(w0), w.E)
    fro, mx = assert_close(bf16_tensor_to_f64(out)[rows], ref, f"T={T} forward (sampled tokens)")
    assert torch.isfinite(out.float()).all()
    print(f"T={T}: forward rows={len(rows)} rel_fro={fro:.2e} rel_max={mx:.2e}")
