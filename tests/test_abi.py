"""The C-ABI library on the host: it loads, exports every function include/stepmoe.h declares,
and rejects bad arguments before touching the GPU. No compute calls (CPU only)."""
import ctypes

import pytest

import sparse_moe_layer_smoe_b200 as smoe


def test_library_exports_every_header_function():
    names = smoe.header_functions()
    assert len(names) >= 14
    L = smoe.lib()
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(smoe._SIGS)


def test_status_strings():
    for code in range(7):
        assert smoe.smoe_status_string(code).startswith(smoe.STATUS[code])
    assert smoe.smoe_status_string(99) == "SMOE_ERR_UNKNOWN"


@pytest.mark.parametrize("field,value,expect", [
    ("hidden", 4000, smoe.SMOE_ERR_UNSUPPORTED),
    ("inter", 1000, smoe.SMOE_ERR_UNSUPPORTED),
    ("shared_inter", 2560, smoe.SMOE_ERR_UNSUPPORTED),
    ("n_experts", 2048, smoe.SMOE_ERR_UNSUPPORTED),
    ("top_k", 33, smoe.SMOE_ERR_UNSUPPORTED),
    ("top_k", 0, smoe.SMOE_ERR_INVALID_ARG),
    ("hidden", -128, smoe.SMOE_ERR_INVALID_ARG),
    ("route_scale", 0.0, smoe.SMOE_ERR_INVALID_ARG),
    ("route_scale", float("inf"), smoe.SMOE_ERR_INVALID_ARG),
    ("swiglu_limit", -1.0, smoe.SMOE_ERR_INVALID_ARG),
    ("swiglu_limit", float("nan"), smoe.SMOE_ERR_INVALID_ARG),
    ("swiglu_limit_shared", float("inf"), smoe.SMOE_ERR_INVALID_ARG),
    ("swiglu_limit", 7.0, smoe.SMOE_OK),
])
def test_config_validation(field, value, expect):
    c = smoe.config()
    setattr(c, field, value)
    assert smoe.smoe_check_config(c) == expect


def test_step_and_tiny_configs_supported():
    assert smoe.smoe_check_config(smoe.config()) == 0
    assert smoe.smoe_check_config(smoe.config(512, 32, 4, 128, 128)) == 0
    small = smoe.config(512, 32, 4, 128, 128)
    small.top_k = 32
    small.n_experts = 31
    assert smoe.smoe_check_config(small) == smoe.SMOE_ERR_UNSUPPORTED


def test_sizes():
    c = smoe.config()
    assert smoe.smoe_packed_weight_bytes(c) == 289 * 3 * 4096 * 1280 * 2
    s1, s8 = smoe.smoe_scratch_bytes(c, 1), smoe.smoe_scratch_bytes(c, 8192)
    w8 = smoe.smoe_workspace_bytes(c, 8192)
    assert 0 < s1 < s8 < w8
    # forward workspace at T=8192 (large token tiles) holds x_perm and y; at T=64 (rows gathered
    # from x inside the GEMM) no x_perm
    assert w8 >= 8192 * 8 * 4096 * 2 + (8192 * 9) * 4096 * 2
    w64 = smoe.smoe_workspace_bytes(c, 64)
    assert w64 < 64 * 8 * 4096 * 2 + (64 * 9) * 4096 * 2 + smoe.smoe_scratch_bytes(c, 64)
    assert smoe.smoe_workspace_bytes(c, 0) > 0


def test_argument_errors_before_any_launch():
    L = smoe.lib()
    c = smoe.config()
    cp = ctypes.byref(c)
    # T < 0, null pointers, misaligned pointers: rejected on the host
    assert L.smoe_route(cp, 16, -1, 16, 16, 16, 16, None, 256, 1 << 20, None) == smoe.SMOE_ERR_INVALID_ARG
    assert L.smoe_route(cp, None, 4, 16, 16, 16, 16, None, 256, 1 << 20, None) == smoe.SMOE_ERR_INVALID_ARG
    assert L.smoe_route(cp, 18, 4, 16, 16, 16, 16, None, 256, 1 << 20, None) == smoe.SMOE_ERR_INVALID_ARG
    assert L.smoe_permute(cp, None, 4, None, 16, 16, 16, 16, None, 256, 1 << 20, None) == smoe.SMOE_ERR_INVALID_ARG
    assert L.smoe_combine(cp, 16, 16, 16, 4, None, 256, 1 << 20, None) == smoe.SMOE_ERR_INVALID_ARG
    assert L.smoe_forward(cp, 16, 4, 16, 16, None, 16, 256, 1 << 30, None) == smoe.SMOE_ERR_INVALID_ARG
    # neither x_perm nor row_token: nothing to read the routed rows from
    assert L.smoe_expert_ffn(cp, 16, None, None, 16, 4, 16, 16, 256, 1 << 30, None) == smoe.SMOE_ERR_INVALID_ARG
    assert L.smoe_pack_weights(cp, 16, 16, 16, 16, 16, None, 16, None) == smoe.SMOE_ERR_INVALID_ARG
    # T == 0 is a no-op
    assert L.smoe_forward(cp, None, 0, None, None, None, None, None, 0, None) == 0
    # a bad config is reported before anything else
    bad = smoe.config(hidden=100)
    assert L.smoe_forward(ctypes.byref(bad), 16, 4, 16, 16, 16, 16, 256, 1 << 30, None) == smoe.SMOE_ERR_UNSUPPORTED


def test_forward_diag_argument_errors():
    L = smoe.lib()
    c = smoe.config()
    cp = ctypes.byref(c)
    fneed = smoe.smoe_workspace_bytes(c, 64)
    good = smoe.SmoeDiag(16, 16, 16, 16, 16)
    # no diag struct, a missing array, a misaligned array: rejected before any launch
    assert L.smoe_forward_diag(cp, 16, 64, 16, 16, 16, 16, None, 256, fneed, None) == smoe.SMOE_ERR_INVALID_ARG
    for i, f in enumerate(smoe.DIAG_FIELDS):
        for bad_ptr in (None, 24):
            d = smoe.SmoeDiag(*[bad_ptr if j == i else 16 for j in range(len(smoe.DIAG_FIELDS))])
            assert L.smoe_forward_diag(cp, 16, 64, 16, 16, 16, 16, ctypes.byref(d), 256, fneed,
                                       None) == smoe.SMOE_ERR_INVALID_ARG, f
    # the forward's own checks still apply (workspace too small), and T == 0 is a no-op
    assert L.smoe_forward_diag(cp, 16, 64, 16, 16, 16, 16, ctypes.byref(good), 256, fneed - 1,
                               None) == smoe.SMOE_ERR_WORKSPACE
    z = smoe.SmoeDiag(16, 16, 16, None, 16)
    assert L.smoe_forward_diag(cp, None, 0, None, None, None, None, ctypes.byref(z), None, 0, None) == 0


def test_fp8_entry_points_argument_errors_and_sizes():
    L = smoe.lib()
    c = smoe.config()
    cp = ctypes.byref(c)
    # packed e4m3 size: one byte per weight + one fp32 scale per weight row, each part 256-aligned
    E1, H, I = 289, 4096, 1280
    al = lambda n: (n + 255) // 256 * 256
    assert smoe.smoe_packed_weight_bytes_fp8(c) == al(E1 * 2 * I * H) + al(E1 * H * I) + al(E1 * 2 * I * 4) + al(E1 * H * 4)
    assert smoe.smoe_workspace_bytes_fp8(c, 64) > smoe.smoe_workspace_bytes(c, 64)
    assert L.smoe_pack_weights_fp8(cp, 16, 16, 16, 16, 16, None, 16, None) == smoe.SMOE_ERR_INVALID_ARG
    assert L.smoe_pack_weights_fp8(cp, 16, 16, 16, 16, 16, 16, 24, None) == smoe.SMOE_ERR_INVALID_ARG
    need = smoe.smoe_workspace_bytes_fp8(c, 64)
    assert L.smoe_forward_fp8(cp, 16, 64, 16, 16, None, 16, 256, need, None) == smoe.SMOE_ERR_INVALID_ARG
    # the bf16 forward's workspace is too small for the e4m3 forward
    assert L.smoe_forward_fp8(cp, 16, 64, 16, 16, 16, 16, 256, smoe.smoe_workspace_bytes(c, 64),
                              None) == smoe.SMOE_ERR_WORKSPACE
    assert L.smoe_forward_fp8(cp, None, 0, None, None, None, None, None, 0, None) == 0
    bad = smoe.config(inter=192)
    assert L.smoe_forward_fp8(ctypes.byref(bad), 16, 4, 16, 16, 16, 16, 256, 1 << 30, None) == smoe.SMOE_ERR_UNSUPPORTED


def test_selftest_argument_checks():
    L = smoe.lib()
    assert L.smoe_selftest_wait_timeout(0, None, 256, None) == smoe.SMOE_ERR_INVALID_ARG
    assert L.smoe_selftest_wait_timeout(2_000_000_000, None, 256, None) == smoe.SMOE_ERR_INVALID_ARG
    assert L.smoe_selftest_wait_timeout(1000, None, None, None) == smoe.SMOE_ERR_INVALID_ARG
    assert L.smoe_selftest_wait_timeout(1000, None, 272, None) == smoe.SMOE_ERR_INVALID_ARG
    assert L.smoe_selftest_wait_timeout(1000, 12, 256, None) == smoe.SMOE_ERR_INVALID_ARG


def test_workspace_checks():
    L = smoe.lib()
    c = smoe.config()
    cp = ctypes.byref(c)
    need = smoe.smoe_scratch_bytes(c, 64)
    # misaligned workspace, then too small
    assert L.smoe_route(cp, 16, 64, 16, 16, 16, 16, None, 272, need, None) == smoe.SMOE_ERR_INVALID_ARG
    assert L.smoe_route(cp, 16, 64, 16, 16, 16, 16, None, 256, need - 1, None) == smoe.SMOE_ERR_WORKSPACE
    fneed = smoe.smoe_workspace_bytes(c, 64)
    assert L.smoe_forward(cp, 16, 64, 16, 16, 16, 16, 256, fneed - 1, None) == smoe.SMOE_ERR_WORKSPACE
    assert L.smoe_combine(cp, 16, 16, 16, 4, 16, 256, 255, None) == smoe.SMOE_ERR_WORKSPACE


def test_noalloc_scratch_size_matches_the_header():
    import re
    text = open(smoe.HEADER).read()
    m = re.search(r"#define SMOE_NOALLOC_SCRATCH_BYTES \((\d+)u << (\d+)\)", text)
    assert m and int(m.group(1)) << int(m.group(2)) == smoe.SMOE_NOALLOC_SCRATCH_BYTES
