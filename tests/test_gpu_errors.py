"""Device-side failure handling, made on the host: bad index data is fed to the library's
kernels, which must skip it (never dereference it), record SMOE_ERR_DEVICE in the workspace's
error word, and leave the rest of the result intact. Nothing here faults, traps or hangs a GPU:
every index is range-checked in the kernel before use."""
import numpy as np
import pytest

import oracle
import synth
from layer_fixtures import cfg_of, device_inputs, host_route

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import sparse_moe_layer_smoe_b200 as smoe  # noqa: E402


def _permute(cfg, idx_np, T):
    k, E = cfg.top_k, cfg.n_experts
    out = dict(counts=torch.empty(E, dtype=torch.int32, device="cuda"),
               offsets=torch.empty(E + 1, dtype=torch.int32, device="cuda"),
               perm_row=torch.empty(T * k, dtype=torch.int32, device="cuda"),
               row_token=torch.empty(T * k, dtype=torch.int32, device="cuda"))
    ws = smoe.workspace(cfg, T, forward=False)
    smoe.smoe_permute(cfg, torch.from_numpy(idx_np).cuda(), T, None, out["counts"], out["offsets"], out["perm_row"],
                      out["row_token"], None, ws)
    return {k2: v.cpu().numpy() for k2, v in out.items()}, smoe.smoe_get_device_error(ws), ws


@pytest.mark.parametrize("T", [64, 2000])   # single-CTA path and multi-block path
@pytest.mark.parametrize("bad", ["out_of_range", "negative", "duplicate"])
def test_permute_skips_bad_expert_ids(T, bad):
    w = synth.WORKLOADS["tiny"]
    cfg = cfg_of(w)
    rng = np.random.default_rng(T)
    idx = np.stack([rng.permutation(w.E)[: w.k] for _ in range(T)]).astype(np.int32)
    t_bad = T // 2
    if bad == "out_of_range":
        idx[t_bad, 1] = w.E + 7
    elif bad == "negative":
        idx[t_bad, 1] = -3
    else:
        idx[t_bad, 1] = idx[t_bad, 0]
    r, code, ws = _permute(cfg, idx, T)
    assert code == smoe.SMOE_ERR_DEVICE
    assert r["perm_row"][t_bad * w.k + 1] == -1
    # every valid entry is placed exactly as the oracle places the valid entries
    good = np.ones(T * w.k, dtype=bool)
    good[t_bad * w.k + 1] = False
    assert r["offsets"][-1] == good.sum()
    rows = r["perm_row"][good]
    assert sorted(rows.tolist()) == list(range(good.sum()))
    flat = idx.reshape(-1)
    e_of_row = np.empty(good.sum(), dtype=np.int64)
    e_of_row[rows] = flat[good]
    assert np.all(np.diff(e_of_row) >= 0)                       # expert-major
    assert np.array_equal(r["counts"], np.bincount(flat[good], minlength=w.E))
    # the error word stays set until cleared, and clears
    smoe.smoe_clear_device_error(ws)
    assert smoe.smoe_get_device_error(ws) == 0


def test_combine_skips_rows_out_of_range():
    w = synth.WORKLOADS["tiny"]
    cfg = cfg_of(w)
    T, k = w.T, w.k
    r = host_route("tiny")
    _, _, perm_row, _ = oracle.permute(r.idx, w.E)
    bad = perm_row.copy()
    bad[5] = T * k + 3          # past the routed rows
    bad[9] = -1                 # a skipped entry
    yh = synth.host_bf16((T * k + T) * w.H, 5, 98, 1.0).reshape(T * k + T, w.H)
    y = torch.from_numpy(yh.view(np.int16)).cuda().view(torch.bfloat16)
    wt = torch.from_numpy(r.w.astype(np.float32)).cuda()
    out = torch.empty(T, w.H, dtype=torch.bfloat16, device="cuda")
    ws = smoe.workspace(cfg, T, forward=False)
    smoe.smoe_combine(cfg, y, torch.from_numpy(bad).cuda(), wt, T, out, ws)
    assert smoe.smoe_get_device_error(ws) == smoe.SMOE_ERR_DEVICE
    assert torch.isfinite(out.float()).all()
    # tokens without a bad entry are unaffected
    ok = torch.empty_like(out)
    ws2 = smoe.workspace(cfg, T, forward=False)
    smoe.smoe_combine(cfg, y, torch.from_numpy(perm_row).cuda(), wt, T, ok, ws2)
    assert smoe.smoe_get_device_error(ws2) == 0
    same = [t for t in range(T) if t not in (5 // k, 9 // k)]
    assert torch.equal(out[same].view(torch.int16), ok[same].view(torch.int16))


def test_expert_ffn_rejects_corrupt_offsets_and_still_runs_the_shared_expert():
    w, x, _, _, packed = device_inputs("tiny")
    cfg = cfg_of(w)
    T, k, E = w.T, w.k, w.E
    r = host_route("tiny")
    _, offsets, _, row_token = oracle.permute(r.idx, E)
    good_y = torch.empty(T * k + T, w.H, dtype=torch.bfloat16, device="cuda")
    ws = smoe.workspace(cfg, T, forward=False)
    smoe.smoe_expert_ffn(cfg, x, None, torch.from_numpy(row_token).cuda(), torch.from_numpy(offsets).cuda(), T,
                         packed, good_y, ws)
    assert smoe.smoe_get_device_error(ws) == 0
    bad_off = offsets.copy()
    bad_off[3], bad_off[4] = bad_off[4] + 5, bad_off[3]      # not monotone
    y = torch.zeros(T * k + T, w.H, dtype=torch.bfloat16, device="cuda")
    ws2 = smoe.workspace(cfg, T, forward=False)
    smoe.smoe_expert_ffn(cfg, x, None, torch.from_numpy(row_token).cuda(), torch.from_numpy(bad_off).cuda(), T,
                         packed, y, ws2)
    assert smoe.smoe_get_device_error(ws2) == smoe.SMOE_ERR_DEVICE
    # routed work dropped (rows untouched), shared rows computed exactly as before
    assert torch.count_nonzero(y[: T * k].float()) == 0
    assert torch.equal(y[T * k:].view(torch.int16), good_y[T * k:].view(torch.int16))
    # the context is still usable
    smoe.smoe_expert_ffn(cfg, x, None, torch.from_numpy(row_token).cuda(), torch.from_numpy(offsets).cuda(), T,
                         packed, y, ws)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), good_y.view(torch.int16))


def test_bounded_wait_times_out_and_the_context_stays_usable():
    """The bounded mbarrier wait of the GEMM roles, run on a barrier nothing arrives at with a
    50 ms limit: it gives up, records SMOE_ERR_TIMEOUT and returns; the layer then still runs."""
    w, x, wr, bias, packed = device_inputs("tiny")
    cfg = cfg_of(w)
    ws = smoe.workspace(cfg, w.T)
    elapsed = torch.zeros(1, dtype=torch.int64, device="cuda")
    smoe.smoe_selftest_wait_timeout(50_000_000, elapsed, ws)
    assert smoe.smoe_get_device_error(ws) == smoe.SMOE_ERR_TIMEOUT
    assert 50_000_000 <= int(elapsed.item()) < 1_000_000_000
    smoe.smoe_clear_device_error(ws)
    out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
    smoe.smoe_forward(cfg, x, w.T, wr, bias, packed, out, ws)
    assert smoe.smoe_get_device_error(ws) == 0
    assert torch.isfinite(out.float()).all()
