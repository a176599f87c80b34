"""GPU parity of the e4m3 (FP8) expert path against the FP8 oracle (oracle/fp8.py).

* smoe_pack_weights_fp8: codes and scales bit-exact against the oracle's quantiser, for whole
  experts of the tiny layer and of the Step shape (the same warp routine quantises x and h);
* smoe_forward_fp8: the layer vs the oracle's e4m3 layer within the layer tolerances (relative
  Frobenius <= 1e-2, max |err| <= 2e-2 max|ref|): all tokens of the tiny layer, >= 256 tokens
  spread over the batch (spike rows included) at decode (gather mode), MTP, prefill and the Zipf-skewed batch (CTA
  pairs, permuted e4m3 rows; skewed mixes 1-row and multi-tile groups), and 128 tokens of a
  1024-token batch (CTA pairs with 64-token tiles);
  the quantisation error against the bf16 oracle is printed for reference;
* deterministic: two calls give the same bits.
"""
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest

import oracle
import synth
from layer_fixtures import (HostExperts, assert_close, bf16_tensor_to_f64, cfg_of, device_inputs, host_route, host_x64,
                            stratified_tokens)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import sparse_moe_layer_smoe_b200 as smoe  # noqa: E402

RNG = np.random.default_rng(88)
_PACKED = {}


def _packed_fp8(w):
    key = (w.H, w.E, w.I)
    if key not in _PACKED:
        _PACKED.clear()
        experts = synth.dev_experts(w)
        _PACKED[key] = smoe.pack_weights_fp8(cfg_of(w), *experts)
        torch.cuda.synchronize()
        del experts
        torch.cuda.empty_cache()
    return _PACKED[key]


def _unpack(w, buf):
    """Host view of the packed e4m3 buffer: per expert gate/up/down codes and scales."""
    E1, H, I = w.E + 1, w.H, w.I
    b = buf.cpu().numpy()
    al = lambda n: (n + 255) // 256 * 256
    o_gu, o_dn = 0, al(E1 * 2 * I * H)
    o_gs = o_dn + al(E1 * H * I)
    o_ds = o_gs + al(E1 * 2 * I * 4)
    gu = b[o_gu:o_gu + E1 * 2 * I * H].reshape(E1, I // 128, H // 128, 256, 128)
    dn = b[o_dn:o_dn + E1 * H * I].reshape(E1, H // 128, I // 128, 128, 128)
    gs = b[o_gs:o_gs + E1 * 2 * I * 4].view(np.float32).reshape(E1, 2, I)
    ds = b[o_ds:o_ds + E1 * H * 4].view(np.float32).reshape(E1, H)

    def expert(g):
        t = gu[g].transpose(0, 2, 1, 3).reshape(I // 128, 256, H)
        gate, up = t[:, :128].reshape(I, H), t[:, 128:].reshape(I, H)
        down = dn[g].transpose(0, 2, 1, 3).reshape(H, I)
        return gate, up, down, gs[g, 0], gs[g, 1], ds[g]
    return expert


@pytest.mark.parametrize("name,groups", [("tiny", [0, 13, 31, 32]), ("decode", [5, 288])])
def test_pack_fp8_codes_and_scales_bit_exact(name, groups):
    w = synth.WORKLOADS[name]
    unpack = _unpack(w, _packed_fp8(w))
    for g in groups:
        Wg, Wu, Wd = (oracle.bf16_to_f64(a) for a in synth.host_expert(w, g))
        gate, up, down, sg, su, sd = unpack(g)
        for codes, scales, W, what in ((gate, sg, Wg, "gate"), (up, su, Wu, "up"), (down, sd, Wd, "down")):
            q, s = oracle.quantize_rows(W)
            assert np.array_equal(scales.view(np.uint32), s.view(np.uint32)), f"expert {g} {what} scales"
            expect = oracle.e4m3_code(q)
            bad = np.nonzero(codes != expect)
            assert bad[0].size == 0, f"expert {g} {what}: {bad[0].size} codes differ, first at {bad[0][0]},{bad[1][0]}"


def _forward_fp8(name, x=None, T=None):
    w, x0, wr, bias, _ = device_inputs(name)
    x = x0 if x is None else x
    T = w.T if T is None else T
    cfg = cfg_of(w)
    packed = _packed_fp8(w)
    ws = smoe.workspace(cfg, T, fp8=True)
    out = torch.empty(T, w.H, dtype=torch.bfloat16, device="cuda")
    smoe.smoe_forward_fp8(cfg, x, T, wr, bias, packed, out, ws)
    assert smoe.smoe_get_device_error(ws) == 0
    return w, out


# The oracle's quantisation of each expert, kept across the tests as uint8 codes and fp32 row
# scales (the Step-shape workloads share their weights): each expert is quantised once, not once
# per test.
_QCACHE = {}
_DECODE = oracle.e4m3_decode(np.arange(256, dtype=np.uint8))


def _quant_expert(w, e):
    key = (w.H, w.E, w.I, w.seed, e)
    if key not in _QCACHE:
        qe = oracle.quantize_expert(*(oracle.bf16_to_f64(a) for a in synth.host_expert(w, e)))
        _QCACHE[key] = tuple(oracle.e4m3_code(v) if i % 2 == 0 else v for i, v in enumerate(qe))
    c = _QCACHE[key]
    return oracle.QuantExpert(tuple(_DECODE[v] if i % 2 == 0 else v for i, v in enumerate(c)))


def _oracle_rows(name, rows, w):
    r = host_route(name)
    x64 = host_x64(name)
    sub = oracle.Route(r.logits[rows], r.s[rows], r.bhat[rows], r.idx[rows], r.w[rows], r.gap[rows])
    lim = dict(limit=w.swiglu_limit, limit_shared=w.swiglu_limit_shared)
    # quantise the experts these rows need on a few host threads first (numpy releases the GIL
    # in the large array operations); the oracle then takes them in its own order
    need = sorted(set(np.unique(sub.idx).tolist()) | {w.E})
    with ThreadPoolExecutor(max_workers=8) as pool:
        list(pool.map(lambda e: _quant_expert(w, e), need))
    ref8 = oracle.moe_sparse_fp8(x64[rows], sub, lambda e: _quant_expert(w, e), w.E, **lim)
    # the bf16 oracle on the same rows, only to print the size of the quantisation error
    ref16 = oracle.moe_sparse(x64[rows], sub, HostExperts(w, cap=24), w.E, **lim) if w.T <= 64 else None
    return ref8, ref16


@pytest.mark.parametrize("name", ["tiny", "decode", "mtp", "prefill", "skewed"])
def test_forward_fp8_parity(name):
    w, out = _forward_fp8(name)
    r = host_route(name)
    if name == "tiny":
        rows = [t for t in range(w.T) if not r.near_tie[t]]
    else:
        cand = [t for t in range(w.T) if not r.near_tie[t]]
        rows = {t for t in stratified_tokens(w.T, 256, RNG) if not r.near_tie[t]} | {cand[0], cand[-1]}
        rows |= {t for t in synth.spike_rows(w).tolist() if not r.near_tie[t]}
        rows = sorted(rows)
    ref8, ref16 = _oracle_rows(name, rows, w)
    got = bf16_tensor_to_f64(out)[rows]
    fro, mx = assert_close(got, ref8, f"{name} e4m3 forward vs e4m3 oracle")
    assert torch.isfinite(out.float()).all()
    q = f"; e4m3 oracle vs bf16 oracle rel_fro={np.linalg.norm(ref8 - ref16) / np.linalg.norm(ref16):.2e}" \
        if ref16 is not None else ""
    print(f"{name}: e4m3 forward rows={len(rows)} rel_fro={fro:.2e} rel_max={mx:.2e}{q}")


def test_forward_fp8_deterministic_and_ragged():
    _, a = _forward_fp8("mtp")
    _, b = _forward_fp8("mtp")
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    # a ragged batch: the first 37 tokens of the decode batch
    w, x, *_ = device_inputs("decode")
    _, c = _forward_fp8("decode", x=x[:37].contiguous(), T=37)
    assert torch.isfinite(c.float()).all()


def test_forward_fp8_mid_batch():
    """T = 1024 (the first tokens of the prefill batch): the e4m3 GEMMs on CTA pairs with 64-token
    tiles, every drain warp taking one or two 32-column chunks; 128 tokens spread over the batch
    against the e4m3 oracle."""
    T = 1024
    w0 = synth.WORKLOADS["prefill"]
    w = synth.Workload("mid_fp8", T, w0.H, w0.E, w0.k, w0.I, w0.Is)
    cfg = cfg_of(w)
    _, _, wr, _, _ = device_inputs("prefill")
    xh = synth.host_x_rows(w0, np.arange(T))
    x = torch.from_numpy(xh.view(np.int16)).cuda().view(torch.bfloat16)
    bias = torch.zeros(w.E, dtype=torch.float32, device="cuda")
    out = torch.empty(T, w.H, dtype=torch.bfloat16, device="cuda")
    ws = smoe.workspace(cfg, T, fp8=True)
    smoe.smoe_forward_fp8(cfg, x, T, wr, bias, _packed_fp8(w0), out, ws)
    assert smoe.smoe_get_device_error(ws) == 0
    x64 = oracle.bf16_to_f64(xh)
    r = oracle.route(x64, oracle.f32_to_f64(synth.host_w_router(w0)), np.zeros(w.E), w.k, w.route_scale)
    rows = sorted(t for t in stratified_tokens(T, 128, RNG) if not r.near_tie[t])
    sub = oracle.Route(r.logits[rows], r.s[rows], r.bhat[rows], r.idx[rows], r.w[rows], r.gap[rows])
    need = sorted(set(np.unique(sub.idx).tolist()) | {w.E})
    with ThreadPoolExecutor(max_workers=8) as pool:
        list(pool.map(lambda e: _quant_expert(w0, e), need))
    ref8 = oracle.moe_sparse_fp8(x64[rows], sub, lambda e: _quant_expert(w0, e), w.E)
    fro, mx = assert_close(bf16_tensor_to_f64(out)[rows], ref8, f"T={T} e4m3 forward vs e4m3 oracle")
    assert torch.isfinite(out.float()).all()
    print(f"T={T}: e4m3 forward rows={len(rows)} rel_fro={fro:.2e} rel_max={mx:.2e}")
