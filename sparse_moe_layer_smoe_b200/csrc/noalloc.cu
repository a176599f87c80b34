// smoe_route_noalloc: the router without a caller-provided workspace.
//
// Some callers cannot allocate device memory at all: a plugin inside an inference runtime
// that is handed only its input and output buffers, or a latency-critical serving path where
// cudaMalloc (which may synchronise the device and take milliseconds) is forbidden once the
// process has started. This entry point needs no workspace: the router's scratch (its K-split
// partial logits) lives in a file-scope device array of SMOE_NOALLOC_SCRATCH_BYTES, which every
// GPU that loads the library holds until the process exits.
//
// In host code the array's name is only a host-side stand-in, never a device address, so its
// device address is looked up here once per device with cudaGetSymbolAddress (the lookup runs
// on the first call made with that device current) and passed to the kernels.
#include <mutex>

#include "internal.h"

namespace smoe {
namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[SMOE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDev = 64;
void* g_scratch_ptr[kMaxDev] = {nullptr};
std::mutex g_scratch_mu;

// Device address of the static scratch on the current device (looked up once per device).
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace smoe

using namespace smoe;

extern "C" smoe_status_t smoe_route_noalloc(const smoe_config_t* c, const smoe_bf16_t* x, int64_t T,
                                            const float* w_router, const float* bias, int32_t* topk_idx,
                                            float* topk_w, float* logits_opt, void* stream) {
    smoe_status_t st = smoe_check_config(c);
    if (st != SMOE_OK) return st;
    if (T < 0) return SMOE_ERR_INVALID_ARG;
    if (T > (int64_t)0x7FFFFFFF / (c->top_k + 1)) return SMOE_ERR_UNSUPPORTED;
    launches_reset();
    if (T == 0) return SMOE_OK;
    const void* req[] = {x, w_router, bias, topk_idx, topk_w};
    for (const void* p : req)
        if (p == nullptr || !aligned16(p)) return SMOE_ERR_INVALID_ARG;
    if (logits_opt != nullptr && !aligned16(logits_opt)) return SMOE_ERR_INVALID_ARG;
    const int sms = num_sms_current_device();
    const RouterPlan rp = router_plan(*c, T, sms, /*allow_tc=*/false);
    const size_t need = rp.scratch_bytes;
    if (need > (size_t)SMOE_NOALLOC_SCRATCH_BYTES) return SMOE_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return SMOE_ERR_CUDA;
    // Every element of the partial-logit area the kernels read is written first in the same
    // call, so nothing needs clearing.
    const cudaError_t e = launch_route(*c, x, T, w_router, bias, topk_idx, topk_w, logits_opt,
                                       static_cast<float*>(scratch), nullptr, sms, static_cast<cudaStream_t>(stream),
                                       /*allow_tc=*/false);
    return e == cudaSuccess ? SMOE_OK : SMOE_ERR_CUDA;
}
