"""The seeded input generator: the C host implementation against its numpy restatement,
and the workload recipes (spike rows, Zipf ranks and bias). CPU only."""
import numpy as np
import pytest

import synth


@pytest.mark.parametrize("std,base", [(1.0, 0), (0.02, 123456789), (50.0, 7)])
def test_host_generator_matches_definition(std, base):
    a = synth.host_f32(20000, 0, synth.TID_WR, std, index_base=base)
    b = synth.normal_reference(20000, 0, synth.TID_WR, std, index_base=base)
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    c = synth.host_bf16(20000, 3, synth.TID_WG, std, index_base=base)
    d = synth.f32_to_bf16_bits(synth.normal_reference(20000, 3, synth.TID_WG, std, index_base=base))
    assert np.array_equal(c, d)


def test_generator_moments():
    z = synth.host_f32(2_000_000, 0, synth.TID_X, 1.0)
    assert abs(z.mean()) < 3e-3 and abs(z.std() - 1.0) < 3e-3
    # Irwin-Hall(8): bounded at ~4.9 std, symmetric
    assert np.abs(z).max() < 4.95
    assert abs(np.mean(z ** 3)) < 1e-2


def test_slices_are_independent_of_the_call():
    whole = synth.host_bf16(5000, 0, synth.TID_X, 1.0)
    part = synth.host_bf16(1000, 0, synth.TID_X, 1.0, index_base=2000)
    assert np.array_equal(whole[2000:3000], part)


def test_bf16_rounding_is_nearest_even():
    f = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0], dtype=np.float32)
    bits = synth.f32_to_bf16_bits(f)
    back = synth.bf16_bits_to_f32(bits)
    assert back.tolist() == [1.0, 1.0 + 4 * 2 ** -8, -2.5, 0.0]


def test_workload_recipes():
    mtp = synth.WORKLOADS["mtp"]
    rows = synth.spike_rows(mtp)
    assert len(rows) == 5 and len(set(rows.tolist())) == 5 and rows.max() < mtp.T
    x = synth.host_x_rows(mtp, rows[:1])
    normal = synth.host_x_rows(synth.WORKLOADS["decode"], rows[:1])  # same index, no spike
    xf = synth.bf16_bits_to_f32(x)
    nf = synth.bf16_bits_to_f32(normal)
    assert 40 < np.abs(xf).mean() / np.abs(nf).mean() < 60
    sk = synth.WORKLOADS["skewed"]
    r = synth.zipf_ranks(sk)
    assert sorted(r.tolist()) == list(range(1, sk.E + 1))
    b = synth.host_bias(sk)
    assert (b == -100.0).sum() == synth.ZIPF_DEAD
    assert b[r == 1][0] == 0.0
    assert np.all(np.diff(b[np.argsort(r)][: sk.E - synth.ZIPF_DEAD]) <= 0)
    assert np.all(synth.host_bias(synth.WORKLOADS["prefill"]) == 0.0)


def test_zipf_fixture_is_consistent():
    import json
    with open(synth.ZIPF_FIXTURE) as f:
        fx = json.load(f)
    assert abs(fx["realised_slope"] - fx["target_slope"]) < 0.02
    assert sum(fx["counts_by_rank"]) == fx["T"] * synth.WORKLOADS["skewed"].k
    assert all(c == 0 for c in fx["counts_by_rank"][-synth.ZIPF_DEAD:])
