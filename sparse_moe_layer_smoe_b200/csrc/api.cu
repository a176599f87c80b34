// The C-ABI of libstepmoe (declared in include/stepmoe.h): argument validation on the host,
// workspace layout, and the launch sequence of each call. No call allocates or synchronises
// (except smoe_get_device_error, which reads the device error word).
#include <math.h>

#include <string.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "internal.h"

namespace smoe {

namespace {
thread_local int g_launches = 0;

constexpr int kMaxDevices = 64;
int g_sms[kMaxDevices] = {0};
std::mutex g_sms_mu;
}  // namespace

void launches_reset() { g_launches = 0; }
void launches_add(int n) { g_launches += n; }

namespace {
struct TimingState {
    bool on = false;
    std::vector<cudaEvent_t> ev;   // 2 per slot: start, end
    std::vector<int> kid;          // kernel of each slot
    int used = 0;
} g_timing;

const char* const kNames[K_NUM_KERNELS] = {"router_logits", "router_topk",   "permute_hist",
                                           "permute_scan",  "permute_scatter", "gather_rows",
                                           "expert_gateup", "expert_down",   "combine",
                                           "pack_gateup",   "pack_down",     "router_split",
                                           "router_gemm",   "diag",        "quantize_x",
                                           "quantize_h",    "pack_fp8"};
}  // namespace

const char* kernel_name(int id) { return (id >= 0 && id < K_NUM_KERNELS) ? kNames[id] : "unknown"; }

LaunchTimer::LaunchTimer(KernelId id, cudaStream_t s) : stream(s) {
    if (!g_timing.on || g_timing.used >= (int)g_timing.kid.size()) return;
    slot = g_timing.used++;
    g_timing.kid[slot] = id;
    cudaEventRecord(g_timing.ev[2 * slot], s);
}

LaunchTimer::~LaunchTimer() {
    if (slot >= 0) cudaEventRecord(g_timing.ev[2 * slot + 1], stream);
}

int num_sms_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    std::lock_guard<std::mutex> lk(g_sms_mu);
    if (g_sms[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        g_sms[dev] = n;
    }
    return g_sms[dev];
}

WsLayout ws_layout(const smoe_config_t& c, int64_t T, int num_sms) {
    WsLayout L;
    const int64_t E = c.n_experts, k = c.top_k, H = c.hidden, I = c.inter;
    const int64_t routed = T * k;
    const RouterPlan rp = router_plan(c, T, num_sms);
    const int64_t nblk = (T + kPermuteTokensPerBlock - 1) / kPermuteTokensPerBlock;
    L.err = 0;
    L.scratch = kAlign;
    const size_t route_b = align_up(rp.scratch_bytes);
    const size_t perm_b = 2 * align_up((size_t)nblk * E * 4);
    const size_t h_b = align_up((size_t)(routed + T) * I * 2);
    L.route_partials = L.scratch;
    L.perm_hist = L.scratch;
    L.perm_base = L.scratch + align_up((size_t)nblk * E * 4);
    L.ffn_h = L.scratch;
    L.scratch_end = L.scratch + std::max(route_b, std::max(perm_b, h_b));
    size_t o = L.scratch_end;
    L.topk_idx = o;  o += align_up((size_t)routed * 4);
    L.topk_w = o;    o += align_up((size_t)routed * 4);
    L.counts = o;    o += align_up((size_t)E * 4);
    L.offsets = o;   o += align_up((size_t)(E + 1) * 4);
    L.perm_row = o;  o += align_up((size_t)routed * 4);
    L.row_token = o; o += align_up((size_t)routed * 4);
    // small token tiles: smoe_forward's gate/up GEMM writes the shared expert's rows of h while
    // the routing may still use the scratch union, so its h lies outside the union
    const bool small_tiles = choose_token_tile(c, T) <= kGatherMaxTile;
    L.ffn_h_fwd = small_tiles ? o : L.ffn_h;
    if (small_tiles) o += h_b;
    L.x_perm = o;    // only when smoe_forward materialises the permuted rows (large token tiles)
    if (!small_tiles) o += align_up((size_t)routed * H * 2);
    L.y = o;         o += align_up((size_t)(routed + T) * H * 2);
    L.row_norm = o;  o += align_up((size_t)routed * 4);
    L.total = o;
    return L;
}

// smoe_forward_fp8: the bf16 layout plus the e4m3 activations and their scales (the permuted
// e4m3 rows, when needed, reuse the x_perm region).
WsLayout ws_layout_fp8(const smoe_config_t& c, int64_t T, int num_sms) {
    WsLayout L = ws_layout(c, T, num_sms);
    const int64_t routed = T * c.top_k;
    size_t o = L.total;
    L.x_q = o;  o += align_up((size_t)T * c.hidden);
    L.s_x = o;  o += align_up((size_t)T * 4);
    L.h_q = o;  o += align_up((size_t)(routed + T) * c.inter);
    L.s_h = o;  o += align_up((size_t)(routed + T) * 4);
    L.total = o;
    return L;
}

}  // namespace smoe

using namespace smoe;

namespace {

smoe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? SMOE_OK : SMOE_ERR_CUDA; }

smoe_status_t check_ws(const smoe_config_t* c, int64_t T, const void* ws, size_t ws_bytes, bool forward,
                       bool fp8 = false) {
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0) return SMOE_ERR_INVALID_ARG;
    const WsLayout L = fp8 ? ws_layout_fp8(*c, T, num_sms_current_device()) : ws_layout(*c, T, num_sms_current_device());
    if (ws_bytes < (forward ? L.total : L.scratch_end)) return SMOE_ERR_WORKSPACE;
    return SMOE_OK;
}

template <class T>
T* at(void* ws, size_t off) {
    return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

}  // namespace

extern "C" {

const char* smoe_status_string(smoe_status_t s) {
    switch (s) {
        case SMOE_OK: return "SMOE_OK";
        case SMOE_ERR_INVALID_ARG: return "SMOE_ERR_INVALID_ARG: null, misaligned or negative argument";
        case SMOE_ERR_UNSUPPORTED: return "SMOE_ERR_UNSUPPORTED: shape or option outside the supported set";
        case SMOE_ERR_WORKSPACE: return "SMOE_ERR_WORKSPACE: workspace too small";
        case SMOE_ERR_CUDA: return "SMOE_ERR_CUDA: a CUDA call failed";
        case SMOE_ERR_DEVICE: return "SMOE_ERR_DEVICE: bad index data met on the device";
        case SMOE_ERR_TIMEOUT: return "SMOE_ERR_TIMEOUT: a bounded device wait gave up";
    }
    return "SMOE_ERR_UNKNOWN";
}

smoe_status_t smoe_check_config(const smoe_config_t* c) {
    if (c == nullptr) return SMOE_ERR_INVALID_ARG;
    if (c->hidden <= 0 || c->n_experts <= 0 || c->top_k <= 0 || c->inter <= 0 || c->shared_inter <= 0)
        return SMOE_ERR_INVALID_ARG;
    if (!(c->route_scale > 0.0f) || !isfinite(c->route_scale)) return SMOE_ERR_INVALID_ARG;
    if (!(c->swiglu_limit >= 0.0f) || !isfinite(c->swiglu_limit) || !(c->swiglu_limit_shared >= 0.0f) ||
        !isfinite(c->swiglu_limit_shared))
        return SMOE_ERR_INVALID_ARG;
    if (c->hidden % 128 != 0 || c->inter % 128 != 0 || c->shared_inter != c->inter) return SMOE_ERR_UNSUPPORTED;
    if (c->n_experts > 1024 || c->top_k > 32 || c->top_k > c->n_experts) return SMOE_ERR_UNSUPPORTED;
    if (c->hidden > 32768 || c->inter > 32768) return SMOE_ERR_UNSUPPORTED;
    return SMOE_OK;
}

smoe_status_t smoe_scratch_bytes(const smoe_config_t* c, int64_t T, size_t* bytes) {
    SMOE_TRY(smoe_check_config(c));
    SMOE_TRY(check_T(c, T));
    if (bytes == nullptr) return SMOE_ERR_INVALID_ARG;
    *bytes = ws_layout(*c, T, num_sms_current_device()).scratch_end;
    return SMOE_OK;
}

smoe_status_t smoe_workspace_bytes(const smoe_config_t* c, int64_t T, size_t* bytes) {
    SMOE_TRY(smoe_check_config(c));
    SMOE_TRY(check_T(c, T));
    if (bytes == nullptr) return SMOE_ERR_INVALID_ARG;
    *bytes = ws_layout(*c, T, num_sms_current_device()).total;
    return SMOE_OK;
}

smoe_status_t smoe_workspace_bytes_fp8(const smoe_config_t* c, int64_t T, size_t* bytes) {
    SMOE_TRY(smoe_check_config(c));
    SMOE_TRY(check_T(c, T));
    if (bytes == nullptr) return SMOE_ERR_INVALID_ARG;
    *bytes = ws_layout_fp8(*c, T, num_sms_current_device()).total;
    return SMOE_OK;
}

smoe_status_t smoe_packed_weight_bytes_fp8(const smoe_config_t* c, size_t* bytes) {
    SMOE_TRY(smoe_check_config(c));
    if (bytes == nullptr) return SMOE_ERR_INVALID_ARG;
    *bytes = fp8_layout(*c).total;
    return SMOE_OK;
}

smoe_status_t smoe_pack_weights_fp8(const smoe_config_t* c, const smoe_bf16_t* w_gate, const smoe_bf16_t* w_up,
                                    const smoe_bf16_t* w_down, const smoe_bf16_t* ws_gate, const smoe_bf16_t* ws_up,
                                    const smoe_bf16_t* ws_down, void* packed, void* stream) {
    SMOE_TRY(smoe_check_config(c));
    SMOE_REQUIRE_PTR(w_gate);
    SMOE_REQUIRE_PTR(w_up);
    SMOE_REQUIRE_PTR(w_down);
    SMOE_REQUIRE_PTR(ws_gate);
    SMOE_REQUIRE_PTR(ws_up);
    SMOE_REQUIRE_PTR(ws_down);
    SMOE_REQUIRE_PTR(packed);
    launches_reset();
    return cuda_status(launch_pack_fp8(*c, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, packed,
                                       static_cast<cudaStream_t>(stream)));
}

smoe_status_t smoe_packed_weight_bytes(const smoe_config_t* c, size_t* bytes) {
    SMOE_TRY(smoe_check_config(c));
    if (bytes == nullptr) return SMOE_ERR_INVALID_ARG;
    *bytes = packed_gateup_bytes(*c) + packed_down_bytes(*c);
    return SMOE_OK;
}

smoe_status_t smoe_pack_weights(const smoe_config_t* c, const smoe_bf16_t* w_gate, const smoe_bf16_t* w_up,
                                const smoe_bf16_t* w_down, const smoe_bf16_t* ws_gate, const smoe_bf16_t* ws_up,
                                const smoe_bf16_t* ws_down, void* packed, void* stream) {
    SMOE_TRY(smoe_check_config(c));
    SMOE_REQUIRE_PTR(w_gate);
    SMOE_REQUIRE_PTR(w_up);
    SMOE_REQUIRE_PTR(w_down);
    SMOE_REQUIRE_PTR(ws_gate);
    SMOE_REQUIRE_PTR(ws_up);
    SMOE_REQUIRE_PTR(ws_down);
    SMOE_REQUIRE_PTR(packed);
    launches_reset();
    return cuda_status(launch_pack(*c, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, packed,
                                   static_cast<cudaStream_t>(stream)));
}

smoe_status_t smoe_route(const smoe_config_t* c, const smoe_bf16_t* x, int64_t T, const float* w_router,
                         const float* bias, int32_t* topk_idx, float* topk_w, float* logits_opt, void* ws,
                         size_t ws_bytes, void* stream) {
    SMOE_TRY(smoe_check_config(c));
    SMOE_TRY(check_T(c, T));
    launches_reset();
    if (T == 0) return SMOE_OK;
    SMOE_REQUIRE_PTR(x);
    SMOE_REQUIRE_PTR(w_router);
    SMOE_REQUIRE_PTR(bias);
    SMOE_REQUIRE_PTR(topk_idx);
    SMOE_REQUIRE_PTR(topk_w);
    SMOE_OPTIONAL_PTR(logits_opt);
    SMOE_TRY(check_ws(c, T, ws, ws_bytes, false));
    const int sms = num_sms_current_device();
    const WsLayout L = ws_layout(*c, T, sms);
    return cuda_status(launch_route(*c, x, T, w_router, bias, topk_idx, topk_w, logits_opt,
                                    at<float>(ws, L.route_partials), at<int32_t>(ws, L.err), sms,
                                    static_cast<cudaStream_t>(stream)));
}

smoe_status_t smoe_permute(const smoe_config_t* c, const int32_t* topk_idx, int64_t T, const smoe_bf16_t* x_opt,
                           int32_t* counts, int32_t* offsets, int32_t* perm_row, int32_t* row_token,
                           smoe_bf16_t* x_perm_opt, void* ws, size_t ws_bytes, void* stream) {
    SMOE_TRY(smoe_check_config(c));
    SMOE_TRY(check_T(c, T));
    launches_reset();
    if (T == 0) return SMOE_OK;
    SMOE_REQUIRE_PTR(topk_idx);
    SMOE_REQUIRE_PTR(counts);
    SMOE_REQUIRE_PTR(offsets);
    SMOE_REQUIRE_PTR(perm_row);
    SMOE_REQUIRE_PTR(row_token);
    SMOE_OPTIONAL_PTR(x_opt);
    SMOE_OPTIONAL_PTR(x_perm_opt);
    SMOE_TRY(check_ws(c, T, ws, ws_bytes, false));
    const WsLayout L = ws_layout(*c, T, num_sms_current_device());
    return cuda_status(launch_permute(*c, topk_idx, T, x_opt, counts, offsets, perm_row, row_token, x_perm_opt,
                                      at<int32_t>(ws, L.perm_hist), at<int32_t>(ws, L.perm_base),
                                      at<int32_t>(ws, L.err), static_cast<cudaStream_t>(stream)));
}

smoe_status_t smoe_expert_ffn(const smoe_config_t* c, const smoe_bf16_t* x, const smoe_bf16_t* x_perm,
                              const int32_t* row_token, const int32_t* offsets, int64_t T, const void* packed,
                              smoe_bf16_t* y, void* ws, size_t ws_bytes, void* stream) {
    SMOE_TRY(smoe_check_config(c));
    SMOE_TRY(check_T(c, T));
    launches_reset();
    if (T == 0) return SMOE_OK;
    SMOE_REQUIRE_PTR(x);
    SMOE_OPTIONAL_PTR(x_perm);
    SMOE_OPTIONAL_PTR(row_token);
    if (x_perm == nullptr && row_token == nullptr) return SMOE_ERR_INVALID_ARG;   // one of the two is needed
    SMOE_REQUIRE_PTR(offsets);
    SMOE_REQUIRE_PTR(packed);
    SMOE_REQUIRE_PTR(y);
    SMOE_TRY(check_ws(c, T, ws, ws_bytes, false));
    const int sms = num_sms_current_device();
    const WsLayout L = ws_layout(*c, T, sms);
    return cuda_status(launch_expert_ffn(*c, x, x_perm, row_token, offsets, T, packed, y, at<uint16_t>(ws, L.ffn_h),
                                         at<int32_t>(ws, L.err), sms, static_cast<cudaStream_t>(stream)));
}

smoe_status_t smoe_combine(const smoe_config_t* c, const smoe_bf16_t* y, const int32_t* perm_row,
                           const float* topk_w, int64_t T, smoe_bf16_t* out, void* ws, size_t ws_bytes,
                           void* stream) {
    SMOE_TRY(smoe_check_config(c));
    SMOE_TRY(check_T(c, T));
    launches_reset();
    if (T == 0) return SMOE_OK;
    SMOE_REQUIRE_PTR(y);
    SMOE_REQUIRE_PTR(perm_row);
    SMOE_REQUIRE_PTR(topk_w);
    SMOE_REQUIRE_PTR(out);
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0) return SMOE_ERR_INVALID_ARG;
    if (ws_bytes < kAlign) return SMOE_ERR_WORKSPACE;
    return cuda_status(launch_combine(*c, y, perm_row, topk_w, T, out, at<int32_t>(ws, 0),
                                      static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {

#ifndef SMOE_SHARED_PREWAIT
#define SMOE_SHARED_PREWAIT 1
#endif
constexpr bool kSharedPrewait = SMOE_SHARED_PREWAIT != 0;

smoe_status_t forward_impl(const smoe_config_t* c, const smoe_bf16_t* x, int64_t T, const float* w_router,
                           const float* bias, const void* packed, smoe_bf16_t* out, const smoe_diag_t* diag, void* ws,
                           size_t ws_bytes, void* stream, bool fp8 = false) {
    SMOE_TRY(smoe_check_config(c));
    SMOE_TRY(check_T(c, T));
    launches_reset();
    if (diag != nullptr) {
        SMOE_REQUIRE_PTR(diag->expert_count);
        SMOE_REQUIRE_PTR(diag->expert_norm_mean);
        SMOE_REQUIRE_PTR(diag->expert_norm_max);
        SMOE_REQUIRE_PTR(diag->summary);
        if (T > 0) SMOE_REQUIRE_PTR(diag->token_confidence);
    }
    if (T == 0) return SMOE_OK;
    SMOE_REQUIRE_PTR(x);
    SMOE_REQUIRE_PTR(w_router);
    SMOE_REQUIRE_PTR(bias);
    SMOE_REQUIRE_PTR(packed);
    SMOE_REQUIRE_PTR(out);
    SMOE_TRY(check_ws(c, T, ws, ws_bytes, true, fp8));
    const int sms = num_sms_current_device();
    const WsLayout L = fp8 ? ws_layout_fp8(*c, T, sms) : ws_layout(*c, T, sms);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t* err = at<int32_t>(ws, L.err);
    int32_t* idx = at<int32_t>(ws, L.topk_idx);
    float* w = at<float>(ws, L.topk_w);
    int32_t* offsets = at<int32_t>(ws, L.offsets);
    int32_t* perm_row = at<int32_t>(ws, L.perm_row);
    int32_t* row_token = at<int32_t>(ws, L.row_token);
    uint16_t* y = at<uint16_t>(ws, L.y);
    float* conf = diag != nullptr ? diag->token_confidence : nullptr;
    float* row_norm = diag != nullptr ? at<float>(ws, L.row_norm) : nullptr;
    // e4m3: the top-k kernel also quantises x per token
    uint8_t* x_q = fp8 ? at<uint8_t>(ws, L.x_q) : nullptr;
    float* s_x = fp8 ? at<float>(ws, L.s_x) : nullptr;
    cudaError_t e = launch_route(*c, x, T, w_router, bias, idx, w, nullptr, at<float>(ws, L.route_partials), err,
                                 sms, s, true, conf, x_q, s_x);
    // small token tiles: routed rows are gathered from x inside the expert GEMM (no permuted
    // copy); large tiles: one gather kernel writes x_perm and the GEMM loads whole tiles
    const bool gather = choose_token_tile(*c, T) <= kGatherMaxTile;
    uint16_t* x_perm = gather ? nullptr : at<uint16_t>(ws, L.x_perm);
    if (!fp8) {
        // Small token tiles: the shared expert's gate/up units run in the GEMM before its
        // dependency wait, overlapping the routing. Their inputs are x (this call's input,
        // complete before the router's first kernel passed its own wait) and the packed weights;
        // their output rows of h lie outside the scratch the routing uses. The one-CTA
        // permutation lets the GEMM launch at once to make room for that.
        const bool prewait = gather && kSharedPrewait && shared_prewait_fits(*c, T, sms);
        if (e == cudaSuccess)
            e = launch_permute(*c, idx, T, gather ? nullptr : x, at<int32_t>(ws, L.counts), offsets, perm_row,
                               row_token, x_perm, at<int32_t>(ws, L.perm_hist), at<int32_t>(ws, L.perm_base), err, s,
                               0, prewait);
        if (e == cudaSuccess)
            e = launch_expert_ffn(*c, x, x_perm, row_token, offsets, T, packed, y, at<uint16_t>(ws, L.ffn_h_fwd), err,
                                  sms, s, prewait);
    } else {
        // e4m3: x was quantised per token by the top-k kernel; the permuted copy (large tiles) is
        // of the e4m3 rows, moved by the same gather kernel as 2-byte pairs
        if (e == cudaSuccess)
            e = launch_permute(*c, idx, T, gather ? nullptr : reinterpret_cast<const uint16_t*>(x_q),
                               at<int32_t>(ws, L.counts), offsets, perm_row, row_token, x_perm,
                               at<int32_t>(ws, L.perm_hist), at<int32_t>(ws, L.perm_base), err, s, c->hidden / 2);
        if (e == cudaSuccess)
            e = launch_expert_ffn_fp8(*c, x_q, gather ? nullptr : reinterpret_cast<const uint8_t*>(x_perm), s_x,
                                      row_token, offsets, T, packed, y, at<uint16_t>(ws, L.ffn_h),
                                      at<uint8_t>(ws, L.h_q), at<float>(ws, L.s_h), err, sms, s);
    }
    if (e == cudaSuccess) e = launch_combine(*c, y, perm_row, w, T, out, err, s, row_norm);
    if (e == cudaSuccess && diag != nullptr)
        e = launch_diag(*c, T, row_norm, offsets, conf, diag->expert_count, diag->expert_norm_mean,
                        diag->expert_norm_max, diag->summary, err, s);
    return cuda_status(e);
}

}  // namespace

extern "C" {

smoe_status_t smoe_forward(const smoe_config_t* c, const smoe_bf16_t* x, int64_t T, const float* w_router,
                           const float* bias, const void* packed, smoe_bf16_t* out, void* ws, size_t ws_bytes,
                           void* stream) {
    return forward_impl(c, x, T, w_router, bias, packed, out, nullptr, ws, ws_bytes, stream);
}

smoe_status_t smoe_forward_fp8(const smoe_config_t* c, const smoe_bf16_t* x, int64_t T, const float* w_router,
                               const float* bias, const void* packed_fp8, smoe_bf16_t* out, void* ws, size_t ws_bytes,
                               void* stream) {
    return forward_impl(c, x, T, w_router, bias, packed_fp8, out, nullptr, ws, ws_bytes, stream, true);
}

smoe_status_t smoe_forward_diag(const smoe_config_t* c, const smoe_bf16_t* x, int64_t T, const float* w_router,
                                const float* bias, const void* packed, smoe_bf16_t* out, const smoe_diag_t* diag,
                                void* ws, size_t ws_bytes, void* stream) {
    if (diag == nullptr) return SMOE_ERR_INVALID_ARG;
    return forward_impl(c, x, T, w_router, bias, packed, out, diag, ws, ws_bytes, stream);
}

smoe_status_t smoe_selftest_wait_timeout(uint64_t limit_ns, uint64_t* elapsed_ns_opt, void* ws, void* stream) {
    if (limit_ns == 0 || limit_ns > 1000000000ull) return SMOE_ERR_INVALID_ARG;
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0) return SMOE_ERR_INVALID_ARG;
    if (elapsed_ns_opt != nullptr && (reinterpret_cast<uintptr_t>(elapsed_ns_opt) & 7u) != 0)
        return SMOE_ERR_INVALID_ARG;
    launches_reset();
    return cuda_status(launch_wait_selftest(static_cast<int32_t*>(ws), limit_ns, elapsed_ns_opt,
                                            static_cast<cudaStream_t>(stream)));
}

smoe_status_t smoe_selftest_swiglu(const float* g, const float* u, int64_t n, float* out, void* stream) {
    if (n < 0) return SMOE_ERR_INVALID_ARG;
    launches_reset();
    if (n == 0) return SMOE_OK;
    SMOE_REQUIRE_PTR(g);
    SMOE_REQUIRE_PTR(u);
    SMOE_REQUIRE_PTR(out);
    return cuda_status(launch_swiglu_selftest(g, u, n, out, static_cast<cudaStream_t>(stream)));
}

smoe_status_t smoe_get_device_error(const void* ws, int32_t* code, void* stream) {
    if (ws == nullptr || code == nullptr) return SMOE_ERR_INVALID_ARG;
    int32_t v = 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return SMOE_ERR_CUDA;
    *code = v;
    return SMOE_OK;
}

smoe_status_t smoe_clear_device_error(void* ws, void* stream) {
    if (ws == nullptr) return SMOE_ERR_INVALID_ARG;
    return cuda_status(cudaMemsetAsync(ws, 0, sizeof(int32_t), static_cast<cudaStream_t>(stream)));
}

int32_t smoe_last_launch_count(void) { return g_launches; }

smoe_status_t smoe_timing_begin(int32_t max_launches) {
    if (max_launches <= 0 || g_timing.on) return SMOE_ERR_INVALID_ARG;
    g_timing.ev.assign(2 * (size_t)max_launches, nullptr);
    g_timing.kid.assign((size_t)max_launches, 0);
    for (auto& e : g_timing.ev) {
        if (cudaEventCreate(&e) != cudaSuccess) {
            for (auto& d : g_timing.ev)
                if (d) cudaEventDestroy(d);
            g_timing.ev.clear();
            g_timing.kid.clear();
            return SMOE_ERR_CUDA;
        }
    }
    g_timing.used = 0;
    g_timing.on = true;
    return SMOE_OK;
}

smoe_status_t smoe_timing_end(smoe_kernel_time_t* out, int32_t cap, int32_t* n) {
    if (!g_timing.on) return SMOE_ERR_INVALID_ARG;
    g_timing.on = false;
    float tot[K_NUM_KERNELS] = {0};
    int cnt[K_NUM_KERNELS] = {0};
    smoe_status_t st = SMOE_OK;
    for (int i = 0; i < g_timing.used; ++i) {
        float ms = 0.f;
        if (cudaEventSynchronize(g_timing.ev[2 * i + 1]) != cudaSuccess ||
            cudaEventElapsedTime(&ms, g_timing.ev[2 * i], g_timing.ev[2 * i + 1]) != cudaSuccess) {
            st = SMOE_ERR_CUDA;
            continue;
        }
        tot[g_timing.kid[i]] += ms;
        cnt[g_timing.kid[i]] += 1;
    }
    for (auto& e : g_timing.ev) cudaEventDestroy(e);
    g_timing.ev.clear();
    g_timing.kid.clear();
    g_timing.used = 0;
    int k = 0;
    for (int id = 0; id < K_NUM_KERNELS; ++id) {
        if (cnt[id] == 0) continue;
        if (out != nullptr && k < cap) {
            memset(out[k].name, 0, sizeof(out[k].name));
            strncpy(out[k].name, kNames[id], sizeof(out[k].name) - 1);
            out[k].launches = cnt[id];
            out[k].total_ms = tot[id];
        }
        ++k;
    }
    if (n != nullptr) *n = (cap < k) ? cap : k;
    return st;
}

}  // extern "C"
