"""fp64 CPU oracle for the sparse MoE FFN layer — TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference
leg may import this package. The CUDA library never imports it and shares no code with it.

The layer's oracle is the plain C++17 program ``smoe_oracle.cpp`` (fp64 loops, std::sort,
std::thread; reached through ``oracle.cpp``), exported here under the layer's function names.
``oracle.moe`` is a second, independent restatement in numpy with the same names; the pins in
``tests/test_oracle_pins.py`` run against both, and ``tests/test_oracle_cross.py`` checks that
the two agree. The e4m3 (``oracle.fp8``) and monitoring (``oracle.diag``) extensions are numpy,
pinned in their own test files.
"""
from . import cpp, moe
from .cpp import (bf16_to_f64, combine, f32_to_f64, moe_dense_masked, moe_given_selection, moe_sparse, normalise,
                  permute, route, router_logits, select_topk, sigmoid, silu, swiglu_ffn, swiglu_hidden,
                  valid_selections)
from .diag import SUMMARY_FIELDS, Diagnostics, diagnostics, expert_output_norms, summarise
from .fp8 import (E4M3_MAX, QuantExpert, e4m3_code, e4m3_decode, e4m3_round, moe_sparse_fp8, quantize_expert,
                  quantize_rows, round_bf16, swiglu_ffn_fp8)
from .moe import NEAR_TIE_EPS, Route

__all__ = ["cpp", "moe", "SUMMARY_FIELDS", "Diagnostics", "diagnostics", "expert_output_norms", "summarise",
           "E4M3_MAX", "QuantExpert", "quantize_expert", "e4m3_code", "e4m3_decode", "e4m3_round", "moe_sparse_fp8", "quantize_rows", "round_bf16",
           "swiglu_ffn_fp8", "NEAR_TIE_EPS", "Route", "bf16_to_f64", "combine", "f32_to_f64", "moe_dense_masked",
           "moe_given_selection", "moe_sparse", "normalise", "permute", "route", "router_logits", "select_topk",
           "sigmoid", "silu", "swiglu_ffn", "swiglu_hidden", "valid_selections"]
