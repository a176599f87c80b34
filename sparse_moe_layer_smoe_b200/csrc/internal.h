// Internal interface between the C-ABI entry points (api.cu) and the kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "../../include/stepmoe.h"

namespace smoe {

constexpr size_t kAlign = 256;
constexpr int kPermuteTokensPerBlock = 256;

inline size_t align_up(size_t v, size_t a = kAlign) { return (v + a - 1) / a * a; }

// Argument checks shared by every entry point (host side, before any launch).
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// T: negative -> invalid; so large that the T*k + T rows overflow int32 -> unsupported.
inline smoe_status_t check_T(const smoe_config_t* c, int64_t T) {
    if (T < 0) return SMOE_ERR_INVALID_ARG;
    if (T > (int64_t)0x7FFFFFFF / (c->top_k + 1)) return SMOE_ERR_UNSUPPORTED;
    return SMOE_OK;
}

#define SMOE_TRY(expr)                        \
    do {                                      \
        smoe_status_t _s = (expr);            \
        if (_s != SMOE_OK) return _s;         \
    } while (0)

#define SMOE_REQUIRE_PTR(p)                                                     \
    do {                                                                        \
        if ((p) == nullptr || !smoe::aligned16(p)) return SMOE_ERR_INVALID_ARG; \
    } while (0)

#define SMOE_OPTIONAL_PTR(p)                                                    \
    do {                                                                        \
        if ((p) != nullptr && !smoe::aligned16(p)) return SMOE_ERR_INVALID_ARG; \
    } while (0)

// Router plan for T tokens. CUDA cores: tokens per CTA, experts per CTA, K splits. Tensor cores
// (tc, large T): W_r split into three bf16 pieces in the workspace, token tile nt.
struct RouterPlan {
    int tm, te, kc, splits;
    bool wide;              // the 64-token CUDA-core tile
    bool tc;
    int nt, e_pad;
    size_t scratch_bytes;   // partial logits (+ the split weights when tc)
};
RouterPlan router_plan(const smoe_config_t& c, int64_t T, int num_sms, bool allow_tc = true);

// Workspace: [error word | scratch union | forward intermediates]
struct WsLayout {
    size_t err = 0;
    size_t scratch = 0;          // start of the scratch union
    size_t route_partials = 0;   // [splits][T][E] fp32  (inside the union)
    size_t perm_hist = 0;        // [nblk][E] int32      (inside the union)
    size_t perm_base = 0;        // [nblk][E] int32      (inside the union)
    size_t ffn_h = 0;            // [T*k + T][I] bf16    (inside the union)
    size_t ffn_h_fwd = 0;        // h of smoe_forward: outside the union for small token tiles
    size_t scratch_end = 0;
    size_t topk_idx = 0, topk_w = 0, counts = 0, offsets = 0, perm_row = 0, row_token = 0, x_perm = 0, y = 0;
    size_t row_norm = 0;         // [T*k] fp32 (smoe_forward_diag)
    size_t x_q = 0, s_x = 0, h_q = 0, s_h = 0;   // smoe_forward_fp8 only
    size_t total = 0;
};
WsLayout ws_layout(const smoe_config_t& c, int64_t T, int num_sms);
WsLayout ws_layout_fp8(const smoe_config_t& c, int64_t T, int num_sms);

int num_sms_current_device();

// Per-thread count of kernels enqueued by the last entry point.
void launches_reset();
void launches_add(int n);

// Per-kernel CUDA-event timing (smoe_timing_begin / smoe_timing_end). Each launcher wraps its
// kernel launches in a LaunchTimer; when timing is off this is one branch.
enum KernelId {
    K_ROUTER_LOGITS = 0, K_ROUTER_TOPK, K_PERMUTE_HIST, K_PERMUTE_SCAN, K_PERMUTE_SCATTER, K_GATHER_ROWS,
    K_EXPERT_GATEUP, K_EXPERT_DOWN, K_COMBINE, K_PACK_GATEUP, K_PACK_DOWN, K_ROUTER_SPLIT, K_ROUTER_GEMM,
    K_DIAG, K_QUANT_X, K_QUANT_H, K_PACK_FP8, K_NUM_KERNELS
};
const char* kernel_name(int id);

struct LaunchTimer {
    int slot = -1;
    cudaStream_t stream = nullptr;
    LaunchTimer(KernelId id, cudaStream_t s);
    ~LaunchTimer();   // records the end event after the launch statement(s) in scope
};

#ifndef SMOE_PDL
#define SMOE_PDL 1   // launch the layer's kernels as programmatic dependents (0: plain stream order)
#endif

// Launch as a programmatic dependent of the previous kernel in the stream (see pdl_wait).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = SMOE_PDL ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

cudaError_t launch_route(const smoe_config_t& c, const uint16_t* x, int64_t T, const float* wr, const float* bias,
                         int32_t* topk_idx, float* topk_w, float* logits_opt, float* partials, int32_t* err,
                         int num_sms, cudaStream_t s, bool allow_tc = true, float* conf_opt = nullptr,
                         uint8_t* x_q_opt = nullptr, float* s_x_opt = nullptr);   // x_q: e4m3 x per token

cudaError_t launch_router_gemm(const uint16_t* x, int64_t T, int H, const uint16_t* w_split, int e_pad, int E,
                               float* logits, int nt, int ksplit, int num_sms, cudaStream_t s);

// early_trigger: the one-CTA permutation lets the next kernel launch before its own dependency
// wait (that kernel then overlaps the routing; it still waits for this one's results).
cudaError_t launch_permute(const smoe_config_t& c, const int32_t* topk_idx, int64_t T, const uint16_t* x,
                           int32_t* counts, int32_t* offsets, int32_t* perm_row, int32_t* row_token,
                           uint16_t* x_perm, int32_t* hist, int32_t* base, int32_t* err, cudaStream_t s,
                           int gather_cols = 0,   // row width in 2-byte units for the x_perm gather (0: hidden)
                           bool early_trigger = false);

// Largest token tile of an expert-GEMM launch for T tokens (16..256).
int choose_token_tile(const smoe_config_t& c, int64_t T);

// Whether smoe_forward runs the shared expert's gate/up units before the GEMM's dependency wait.
bool shared_prewait_fits(const smoe_config_t& c, int64_t T, int num_sms);

// smoe_forward reads routed rows straight from x (TMA row gathers) when the largest token tile
// is at most this; above it, per-row gathers cost more than one gather kernel plus tile loads.
#ifndef SMOE_GATHER_MAX_TILE
#define SMOE_GATHER_MAX_TILE 32
#endif
constexpr int kGatherMaxTile = SMOE_GATHER_MAX_TILE;

// x_perm == nullptr selects gather mode: routed rows are read from x through row_token.
// Returns cudaErrorNotSupported when the driver entry point for tensor maps is unavailable.
// shared_prewait (gather mode): the gate/up kernel computes the shared expert's units before its
// dependency wait, so x must not come from the two kernels launched just before it; h must
// not overlap memory those kernels use.
cudaError_t launch_expert_ffn(const smoe_config_t& c, const uint16_t* x, const uint16_t* x_perm,
                              const int32_t* row_token, const int32_t* offsets, int64_t T, const void* packed,
                              uint16_t* y, uint16_t* h, int32_t* err, int num_sms, cudaStream_t s,
                              bool shared_prewait = false);

// row_norm_opt: when set, also ||y[r]||_2 of every routed row r (fp32, [T*k]).
cudaError_t launch_combine(const smoe_config_t& c, const uint16_t* y, const int32_t* perm_row, const float* topk_w,
                           int64_t T, uint16_t* out, int32_t* err, cudaStream_t s, float* row_norm_opt = nullptr);

// Per-expert output-norm statistics and the layer summary of smoe_forward_diag (one CTA).
cudaError_t launch_diag(const smoe_config_t& c, int64_t T, const float* row_norm, const int32_t* offsets,
                        const float* conf, int32_t* count, float* norm_mean, float* norm_max, float* summary,
                        int32_t* err, cudaStream_t s);

cudaError_t launch_pack(const smoe_config_t& c, const uint16_t* wg, const uint16_t* wu, const uint16_t* wd,
                        const uint16_t* sg, const uint16_t* su, const uint16_t* sd, void* packed, cudaStream_t s);

// The bounded-wait self-test (smoe_selftest_wait_timeout).
cudaError_t launch_wait_selftest(int32_t* err, uint64_t limit_ns, uint64_t* elapsed_ns, cudaStream_t s);

// The expert epilogue's SiLU(g) * u (smoe_selftest_swiglu).
cudaError_t launch_swiglu_selftest(const float* g, const float* u, int64_t n, float* out, cudaStream_t s);

size_t packed_gateup_bytes(const smoe_config_t& c);
size_t packed_down_bytes(const smoe_config_t& c);

// ---- e4m3 experts (per-row scales; see smoe_pack_weights_fp8)
struct Fp8Layout {
    size_t gateup = 0, down = 0, gateup_scale = 0, down_scale = 0, total = 0;   // byte offsets, size
};
Fp8Layout fp8_layout(const smoe_config_t& c);

cudaError_t launch_pack_fp8(const smoe_config_t& c, const uint16_t* wg, const uint16_t* wu, const uint16_t* wd,
                            const uint16_t* sg, const uint16_t* su, const uint16_t* sd, void* packed, cudaStream_t s);

// q[r][:] = e4m3(a[r][:] / s[r]), s[r] = max |a[r][:]| / 448 (1 for an all-zero row); one warp per row.
cudaError_t launch_quantize_rows(const uint16_t* a, int64_t rows, int cols, uint8_t* q, float* scale, KernelId id,
                                 cudaStream_t s);

// Gate/up and down with e4m3 operands: x_q [T][H] (+ x_q_perm [T*k][H] or nullptr: gather mode),
// s_x [T]; the SwiGLU hidden h (bf16) is quantised per row into h_q / s_h between the GEMMs.
cudaError_t launch_expert_ffn_fp8(const smoe_config_t& c, const uint8_t* x_q, const uint8_t* x_q_perm,
                                  const float* s_x, const int32_t* row_token, const int32_t* offsets, int64_t T,
                                  const void* packed_fp8, uint16_t* y, uint16_t* h, uint8_t* h_q, float* s_h,
                                  int32_t* err, int num_sms, cudaStream_t s);

}  // namespace smoe
