/*
 * libstepmoe — one sparse MoE FFN layer of the Step 3.5 Flash shape on NVIDIA B200 (sm_100a).
 *
 * The layer (sources by page and section):
 *   - Step-3.5-Flash model card (llm-atlas), raw config fields: hidden_size 4096,
 *     moe_num_experts 288, moe_top_k 8, moe_intermediate_size 1280, share_expert_dim 1280,
 *     norm_expert_weight true, moe_router_activation sigmoid, moe_router_scaling_factor 3,
 *     use_moe_router_bias true, need_fp32_gate true, torch_dtype bfloat16.
 *   - Step 3.5 Flash summary (hyper.ai), section "方法" (method): every MoE layer runs 8 of
 *     288 routed experts per token plus one shared expert.
 *   - Step 3.5 Flash summary (paperlayer.ai), §2.2 "Sparse MoE Backbone with Hybrid
 *     Attention"; §4.1.2 "Expert Collapse Beyond Routing Collapse" (router bias as the
 *     loss-free balancing device); §B "Detail Analysis of Localized Activation Blow-up"
 *     (SwiGLU experts with gate and up projections).
 *
 *   out[t] = F_shared(x_t) + sum_{j<k} w[t,j] * F_{idx[t,j]}(x_t)
 *   F(x)   = W_d (SiLU(W_g x) * (W_u x))
 *   s      = sigmoid(x W_r^T)  in fp32;   idx = top-k of (s + bias);   w = 3 * s_sel / sum(s_sel)
 *
 * Conventions for every call:
 *   - Tensor pointers are DEVICE pointers, owned by the caller, row-major and contiguous,
 *     16-byte aligned (cudaMalloc memory is). bf16 tensors are raw bf16 bit patterns.
 *   - The library allocates and frees nothing. Scratch lives in a caller-owned workspace
 *     whose size smoe_scratch_bytes / smoe_workspace_bytes report; its first 256 bytes hold
 *     the device error word.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream).
 *     They validate arguments on the host, enqueue kernels, and return a status. There is
 *     no host<->device synchronisation inside any call except smoe_get_device_error.
 *   - No exceptions cross the ABI. T == 0 is a no-op returning SMOE_OK.
 *   - Supported shapes: hidden, inter multiples of 128; shared_inter == inter;
 *     1 <= top_k <= min(32, n_experts); n_experts <= 1024.
 *     Anything else returns SMOE_ERR_UNSUPPORTED before any work is enqueued.
 *   - Bad data found on the device (an expert index out of range, a duplicate expert in a
 *     token's selection, a row index out of range) is skipped, never dereferenced, and
 *     recorded in the workspace's device error word (SMOE_ERR_DEVICE). Bounded waits in
 *     the expert GEMM that give up record SMOE_ERR_TIMEOUT. Read with
 *     smoe_get_device_error; the first error recorded wins until smoe_clear_device_error.
 */
#ifndef STEPMOE_H
#define STEPMOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SMOE_API __attribute__((visibility("default")))
#else
#define SMOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SMOE_OK = 0,
    SMOE_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, negative size */
    SMOE_ERR_UNSUPPORTED = 2,   /* shape or option outside the supported set */
    SMOE_ERR_WORKSPACE = 3,     /* workspace smaller than required */
    SMOE_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed */
    SMOE_ERR_DEVICE = 5,        /* (device error word) bad index data met on the device */
    SMOE_ERR_TIMEOUT = 6        /* (device error word) a bounded wait gave up */
} smoe_status_t;

typedef uint16_t smoe_bf16_t;   /* raw bf16 bit pattern */

typedef struct {
    int32_t hidden;        /* H: model width (4096)                         */
    int32_t n_experts;     /* E: routed experts (288)                       */
    int32_t top_k;         /* k: routed experts per token (8)               */
    int32_t inter;         /* I: routed expert intermediate width (1280)    */
    int32_t shared_inter;  /* Is: shared expert intermediate width (1280)   */
    float route_scale;     /* factor applied to the normalised weights (3)  */
    float swiglu_limit;    /* SwiGLU clamp of the routed experts; 0 = off   */
    float swiglu_limit_shared; /* SwiGLU clamp of the shared expert; 0 = off */
} smoe_config_t;
/* SwiGLU clamp (model card raw config fields swiglu_limits, swiglu_limits_shared: 0 for most
 * layers, 7 (routed) and 16 (shared) for the deepest ones; activation clipping against
 * localized activation blow-up, paperlayer.ai summary §4.1.3 and §B). The pages do not spell out
 * the clamp; read here as: with limit L > 0, gate g = min(g, L) and up u = clamp(u, -L, L) before
 * h = SiLU(g) * u. Limits must be finite and >= 0. */

/* Human-readable name of a status code. Never NULL. */
SMOE_API const char* smoe_status_string(smoe_status_t status);

/* Validate a configuration against the supported set (see conventions). */
SMOE_API smoe_status_t smoe_check_config(const smoe_config_t* cfg);

/* Bytes of workspace the per-call entry points (route, permute, expert_ffn, combine) need
 * for T tokens: the error word plus the largest of the calls' scratch areas. */
SMOE_API smoe_status_t smoe_scratch_bytes(const smoe_config_t* cfg, int64_t T, size_t* bytes);

/* Bytes of workspace smoe_forward needs for T tokens: the scratch above plus every
 * intermediate of the layer (selection, permutation, permuted rows, expert outputs). */
SMOE_API smoe_status_t smoe_workspace_bytes(const smoe_config_t* cfg, int64_t T, size_t* bytes);

/* Bytes of the packed expert-weight buffer smoe_pack_weights writes. */
SMOE_API smoe_status_t smoe_packed_weight_bytes(const smoe_config_t* cfg, size_t* bytes);

/* Pack the routed and shared expert weights into the layout the expert GEMMs stream.
 *   w_gate, w_up  [E][I][H] bf16      routed gate / up projections (row = output feature)
 *   w_down        [E][H][I] bf16      routed down projections
 *   ws_gate, ws_up [Is][H] bf16, ws_down [H][Is] bf16   the shared expert
 *   packed        device buffer of smoe_packed_weight_bytes bytes, written here.
 * Packed layout (tile-major: each tile the GEMMs load is contiguous): the gate/up block
 * [(E+1)][I/128][H/64][256][64] (tile (g, mb, kb) = the 128 gate rows of features
 * 128 mb .. 128 mb + 127, then the matching 128 up rows, over K columns 64 kb .. 64 kb + 63;
 * group E = shared expert), followed by the down block [(E+1)][H/128][I/64][128][64].
 * Source: the SwiGLU expert (paperlayer.ai summary, §B) with moe_intermediate_size /
 * share_expert_dim of the model card. Run once per layer. */
SMOE_API smoe_status_t smoe_pack_weights(const smoe_config_t* cfg, const smoe_bf16_t* w_gate, const smoe_bf16_t* w_up,
                                const smoe_bf16_t* w_down, const smoe_bf16_t* ws_gate, const smoe_bf16_t* ws_up,
                                const smoe_bf16_t* ws_down, void* packed, void* stream);

/* Router (model card: need_fp32_gate, moe_router_activation sigmoid, use_moe_router_bias,
 * moe_top_k, norm_expert_weight, moe_router_scaling_factor; paperlayer.ai §4.1.2 for the
 * bias as a selection device).
 *   x         [T][H] bf16 activations
 *   w_router  [E][H] fp32 router weights;  bias [E] fp32 (selection only)
 *   topk_idx  [T][k] int32 out: experts in descending order of s + bias; equal biased
 *             scores order by the larger fp32 logit, then the smaller expert index
 *   topk_w    [T][k] fp32 out: route_scale * s_j / sum_j s_j over the selected UNBIASED s
 *   logits_opt [T][E] fp32 out (fp32 logits) or NULL
 *   ws, ws_bytes  workspace of at least smoe_scratch_bytes(cfg, T)
 * Logits accumulate in fp32 from bf16 x upcast exactly; sigmoid and weights in fp32. */
SMOE_API smoe_status_t smoe_route(const smoe_config_t* cfg, const smoe_bf16_t* x, int64_t T, const float* w_router,
                         const float* bias, int32_t* topk_idx, float* topk_w, float* logits_opt, void* ws,
                         size_t ws_bytes, void* stream);

/* Token -> expert dispatch: per-expert histogram, exclusive scan, stable scatter.
 *   topk_idx  [T][k] int32 (from smoe_route, or any selection of k distinct experts)
 *   counts    [E] int32 out: rows per expert
 *   offsets   [E+1] int32 out: exclusive scan of counts (offsets[E] = T*k when every entry
 *             is valid; skipped entries get perm_row = -1 and no row)
 *   perm_row  [T*k] int32 out: entry t*k+j -> its row; rows are expert-major, then token
 *             ascending, then slot ascending (a unique order, so results are bit-exact)
 *   row_token [T*k] int32 out: row -> token
 *   x_opt, x_perm_opt: when both are non-NULL, x_perm[r] = x[row_token[r]] ([T*k][H] bf16)
 * Out-of-range or duplicate expert ids are skipped and set SMOE_ERR_DEVICE. */
SMOE_API smoe_status_t smoe_permute(const smoe_config_t* cfg, const int32_t* topk_idx, int64_t T, const smoe_bf16_t* x_opt,
                           int32_t* counts, int32_t* offsets, int32_t* perm_row, int32_t* row_token,
                           smoe_bf16_t* x_perm_opt, void* ws, size_t ws_bytes, void* stream);

/* Expert FFNs: grouped gate/up GEMM fused with SiLU-mul, then grouped down GEMM, on the
 * tensor cores (tcgen05, bf16 in, fp32 accumulate). Groups 0..E-1 are the routed experts
 * over their rows; group E is the shared expert over all T rows of x.
 *   x         [T][H] bf16
 *   x_perm    [T*k][H] bf16 rows grouped by offsets, or NULL: then the routed rows are read
 *             straight from x through row_token (TMA row gathers; no permuted copy of x).
 *             The results are the same either way; with token tiles above 32 rows the row
 *             gathers are slower than loading x_perm (smoe_forward builds x_perm there).
 *   row_token [T*k] int32, as written by smoe_permute (needed when x_perm is NULL)
 *   offsets   [E+1] int32 (device), as written by smoe_permute
 *   packed    packed weights (smoe_pack_weights)
 *   y         [T*k + T][H] bf16 out: rows 0..T*k-1 routed (permuted order), rows T*k.. shared
 * The SwiGLU hidden h = SiLU(g) * u is computed in fp32 from fp32 accumulators and rounded
 * once to bf16 (kept in the workspace); y is rounded once to bf16.
 * Returns SMOE_ERR_INVALID_ARG when both x_perm and row_token are NULL. */
SMOE_API smoe_status_t smoe_expert_ffn(const smoe_config_t* cfg, const smoe_bf16_t* x, const smoe_bf16_t* x_perm,
                              const int32_t* row_token, const int32_t* offsets, int64_t T, const void* packed,
                              smoe_bf16_t* y, void* ws, size_t ws_bytes, void* stream);

/* Combine (hyper.ai summary "方法": 8 routed + 1 shared expert per token):
 *   out[t] = y[T*k + t] + sum_{j<k} topk_w[t][j] * y[perm_row[t*k + j]]
 * accumulated in fp32 in slot order j = 0..k-1, shared row added last, rounded once to bf16.
 *   y [T*k + T][H] bf16, perm_row [T*k] int32, topk_w [T][k] fp32, out [T][H] bf16.
 * Rows out of range are skipped and set SMOE_ERR_DEVICE in the workspace's error word. */
SMOE_API smoe_status_t smoe_combine(const smoe_config_t* cfg, const smoe_bf16_t* y, const int32_t* perm_row,
                           const float* topk_w, int64_t T, smoe_bf16_t* out, void* ws, size_t ws_bytes,
                           void* stream);

/* The whole layer: route -> permute -> expert_ffn -> combine on one stream, every
 * intermediate in the workspace (at least smoe_workspace_bytes(cfg, T) bytes). When the mean
 * rows per expert are small (token tiles <= 32 rows) the expert GEMM gathers routed rows from
 * x itself; otherwise permute writes the permuted copy x_perm into the workspace.
 *   x [T][H] bf16, w_router [E][H] fp32, bias [E] fp32, packed weights, out [T][H] bf16. */
SMOE_API smoe_status_t smoe_forward(const smoe_config_t* cfg, const smoe_bf16_t* x, int64_t T, const float* w_router,
                           const float* bias, const void* packed, smoe_bf16_t* out, void* ws, size_t ws_bytes,
                           void* stream);

/* Monitoring outputs of one layer step (smoe_forward_diag), after the Step 3.5 Flash
 * summary (paperlayer.ai): §4.1.2 monitors per-expert activation norms (a falling
 * minimum-to-median ratio warns of expert death), §4.1.3 reads localized activation blow-up
 * from the maximum-to-median activation-norm ratio, §5.2.1 uses routing confidence as a
 * stability proxy. The pages define none of these numerically; the readings here:
 *   expert norm   ||F_e(x_t)||_2, the L2 norm of routed expert e's output row for token t
 *                 (the bf16 row the layer combines, before its routing weight);
 *   confidence    of token t: the mean of its k selected (unbiased) sigmoid scores.
 * All pointers are caller-owned device arrays, 16-byte aligned, written on the stream. */
typedef struct {
    int32_t* expert_count;      /* [E] tokens routed to expert e */
    float* expert_norm_mean;    /* [E] mean expert norm over those tokens (0 when none) */
    float* expert_norm_max;     /* [E] largest expert norm over those tokens (0 when none) */
    float* token_confidence;    /* [T] routing confidence of each token */
    float* summary;             /* [SMOE_DIAG_SUMMARY] the layer summary, indexed below */
} smoe_diag_t;

enum {
    SMOE_DIAG_ACTIVE_EXPERTS = 0,   /* experts that received at least one token */
    SMOE_DIAG_NORM_MEDIAN,          /* median of expert_norm_mean over those experts (mean of the
                                       two middle values for an even count) */
    SMOE_DIAG_NORM_MAX_TO_MEDIAN,   /* their largest expert_norm_mean / the median (0 if median 0) */
    SMOE_DIAG_NORM_MIN_TO_MEDIAN,   /* their smallest expert_norm_mean / the median (0 if median 0) */
    SMOE_DIAG_CONF_MEAN,            /* mean token confidence */
    SMOE_DIAG_CONF_MIN,             /* smallest token confidence */
    SMOE_DIAG_LOAD_MAX_TO_MEAN,     /* largest expert_count / (T * k / E) */
    SMOE_DIAG_NORM_PEAK,            /* largest expert_norm_max */
    SMOE_DIAG_SUMMARY               /* number of summary entries */
};

/* smoe_forward plus the monitoring outputs above (diag must be non-NULL, every array set).
 * Same workspace as smoe_forward; the extra work is a sum of squares per routed row inside
 * the combine kernel, the confidence store in the top-k kernel and one single-CTA kernel.
 * Every output is deterministic. Returns SMOE_ERR_INVALID_ARG for a NULL or misaligned array. */
SMOE_API smoe_status_t smoe_forward_diag(const smoe_config_t* cfg, const smoe_bf16_t* x, int64_t T,
                                const float* w_router, const float* bias, const void* packed, smoe_bf16_t* out,
                                const smoe_diag_t* diag, void* ws, size_t ws_bytes, void* stream);

/* ---- e4m3 (FP8) experts -------------------------------------------------------------------
 * The Step 3.5 Flash summary (paperlayer.ai) fits the model into a 128 GB workstation budget,
 * which calls for low-precision experts, but names no format. The format and quantiser here
 * are readings, and the test oracle implements the same ones:
 *   e4m3 codes (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, largest finite 448),
 *   rounding to nearest even, finite values beyond +-448 saturating;
 *   one fp32 scale per row of a matrix: s = max|row| / 448 (1 for an all-zero row), codes
 *   e4m3(a / s) with a / s in IEEE fp32. Weight rows are output features (gate, up and down
 *   rows of every expert); activation rows are tokens (x) or hidden rows (h).
 * The expert: gate and up accumulate code products in fp32 on the tensor cores and are scaled
 * by s_w * s_x; SiLU(gate) * up (with the SwiGLU clamp) is rounded to bf16 and quantised per
 * row; the down product is scaled by s_w * s_h. Router, combine and shared add as in bf16.
 * Packed layout (tile-major; every tile the GEMMs load is contiguous):
 *   gate/up codes [(E+1)][I/128][H/128][256][128] (tile (g, mb, kb): the 128 gate rows of
 *   features 128 mb .. +127, then the matching 128 up rows, K columns 128 kb .. +127),
 *   down codes [(E+1)][H/128][I/128][128][128], then the fp32 scales: gate/up [(E+1)][2][I]
 *   (gate rows, then up rows), down [(E+1)][H]. Each part starts on a 256-byte boundary. */

/* Bytes of the packed e4m3 expert buffer smoe_pack_weights_fp8 writes. */
SMOE_API smoe_status_t smoe_packed_weight_bytes_fp8(const smoe_config_t* cfg, size_t* bytes);

/* Quantise and pack the experts (same inputs as smoe_pack_weights). Run once per layer. */
SMOE_API smoe_status_t smoe_pack_weights_fp8(const smoe_config_t* cfg, const smoe_bf16_t* w_gate,
                                const smoe_bf16_t* w_up, const smoe_bf16_t* w_down, const smoe_bf16_t* ws_gate,
                                const smoe_bf16_t* ws_up, const smoe_bf16_t* ws_down, void* packed_fp8,
                                void* stream);

/* Workspace bytes of smoe_forward_fp8 for T tokens (smoe_forward's plus the e4m3 activations). */
SMOE_API smoe_status_t smoe_workspace_bytes_fp8(const smoe_config_t* cfg, int64_t T, size_t* bytes);

/* The whole layer with e4m3 experts: route (fp32, as smoe_forward; its top-k kernel also
 * quantises x per token) -> permute -> gate/up (e4m3 tensor cores) -> quantise h per row ->
 * down -> combine. Arguments as
 * smoe_forward, with packed_fp8 from smoe_pack_weights_fp8 and a workspace of at least
 * smoe_workspace_bytes_fp8(cfg, T) bytes. */
SMOE_API smoe_status_t smoe_forward_fp8(const smoe_config_t* cfg, const smoe_bf16_t* x, int64_t T,
                                const float* w_router, const float* bias, const void* packed_fp8,
                                smoe_bf16_t* out, void* ws, size_t ws_bytes, void* stream);

/* Synchronise `stream` and read the workspace's device error word into *code
 * (SMOE_OK when no kernel recorded an error). */
SMOE_API smoe_status_t smoe_get_device_error(const void* ws, int32_t* code, void* stream);

/* Reset the device error word to SMOE_OK (asynchronous on `stream`). */
SMOE_API smoe_status_t smoe_clear_device_error(void* ws, void* stream);

/* Failure-detection self-test: one thread waits, through the bounded mbarrier wait every GEMM
 * role uses, on a barrier nothing arrives at, with the given limit (1 ns .. 1 s). The wait gives
 * up after limit_ns, records SMOE_ERR_TIMEOUT in the workspace's error word (read it with
 * smoe_get_device_error) and the kernel exits normally, leaving the context usable. If
 * elapsed_ns_opt (device, 8-byte aligned) is set, the measured wait is written there. Needs only
 * the workspace's first 256 bytes. Returns SMOE_ERR_INVALID_ARG for a limit outside the range or
 * a misaligned pointer. (A library operation of its own; the pages have no counterpart.) */
SMOE_API smoe_status_t smoe_selftest_wait_timeout(uint64_t limit_ns, uint64_t* elapsed_ns_opt, void* ws, void* stream);

/* Self-test of the expert epilogue's arithmetic: out[i] = SiLU(g[i]) * u[i] for n elements,
 * computed as the gate/up GEMM's epilogue computes it from its fp32 accumulators (fast exponential
 * and reciprocal on the special-function unit). SiLU(z) = z / (1 + e^-z) is the expert
 * activation (Step 3.5 Flash summary, paperlayer.ai, §B: SwiGLU gate and up projections). All
 * pointers are device fp32 arrays of n elements, 16-byte aligned; asynchronous on the stream. */
SMOE_API smoe_status_t smoe_selftest_swiglu(const float* g, const float* u, int64_t n, float* out, void* stream);

/* Number of kernel launches the last successful call on this host thread enqueued. */
SMOE_API int32_t smoe_last_launch_count(void);

/* Per-kernel device time, measured with CUDA events recorded on the launching stream
 * immediately before and after each of the library's kernel launches. */
typedef struct {
    char name[32];       /* kernel: router_logits, router_topk, permute_hist, permute_scan,
                            permute_scatter, gather_rows, expert_gateup, expert_down, combine,
                            pack_gateup, pack_down, router_split, router_gemm, diag,
                            quantize_x, quantize_h, pack_fp8 */
    int32_t launches;    /* launches recorded */
    float total_ms;      /* summed event-to-event time of those launches */
} smoe_kernel_time_t;

/* Start recording: creates 2 * max_launches events up front (no allocation later); launches
 * beyond max_launches are not recorded. Not thread-safe with concurrent library calls. */
SMOE_API smoe_status_t smoe_timing_begin(int32_t max_launches);

/* Stop recording: synchronise the recorded events, write one entry per kernel that ran
 * (at most cap entries) to out, their number to *n, and destroy the events. */
SMOE_API smoe_status_t smoe_timing_end(smoe_kernel_time_t* out, int32_t cap, int32_t* n);

/* Allocation-free router, for callers that cannot allocate device memory: a plugin that an
 * inference runtime hands only its input and output buffers, or a serving path where
 * cudaMalloc is forbidden after start-up because it can synchronise the device and stall.
 * The pages have no counterpart to this entry point; it exists only for such callers.
 * Same arguments, checks and results as smoe_route, without the workspace; it always runs the
 * CUDA-core router kernels. Its scratch (the router's K-split partial logits,
 * splits x T x E x 4 bytes) is a static device array of SMOE_NOALLOC_SCRATCH_BYTES that every
 * GPU loading the library holds until the process exits; a T that needs more returns
 * SMOE_ERR_WORKSPACE before any launch. Large batches run with a K split of 1 (at E = 288 on
 * a 148-SM B200: every batch above 3,136 tokens), so the largest batch is
 * floor(16 MiB / (E x 4)) = 14,563 tokens at E = 288; smaller batches use up to 16 splits and
 * fit too (at most 9.4 MB at E = 288). The array's device address is looked up
 * (cudaGetSymbolAddress) on every call in the current context; the first call on each device
 * or context also loads the library's device code there, so make that first call before any
 * stream capture. Every call shares the one array and keeps nothing from earlier calls:
 * calls that overlap on the GPU (several streams or host threads) race on it, so the caller
 * must serialise them. Allocates and frees nothing. */
#define SMOE_NOALLOC_SCRATCH_BYTES (16u << 20)
SMOE_API smoe_status_t smoe_route_noalloc(const smoe_config_t* cfg, const smoe_bf16_t* x, int64_t T,
                                          const float* w_router, const float* bias, int32_t* topk_idx,
                                          float* topk_w, float* logits_opt, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* STEPMOE_H */
