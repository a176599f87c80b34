// smoe_route_noalloc: the router without a caller-provided workspace.
//
// Some callers cannot allocate device memory at all: a plugin inside an inference runtime
// that is handed only its input and output buffers, or a latency-critical serving path where
// cudaMalloc (which may synchronise the device and take milliseconds) is forbidden once the
// process has started. This entry point needs no workspace: the router's scratch (its K-split
// partial logits) lives in a file-scope device array of SMOE_NOALLOC_SCRATCH_BYTES, which every
// GPU that loads the library holds until the process exits.
//
// In host code the array's name is only a host-side stand-in, never a device address. Its
// device address belongs to the module instance loaded in the current context, so it is looked
// up with cudaGetSymbolAddress on every call, with the caller's device current: a host that
// runs its own (non-primary) contexts, or resets a device and so reloads the module, gets the
// address that is valid now. The first call on each device (or context) is the one that loads
// the module there; after that the lookup is a table read.
#include "internal.h"

namespace smoe {
namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[SMOE_NOALLOC_SCRATCH_BYTES];

}  // namespace
}  // namespace smoe

using namespace smoe;

extern "C" smoe_status_t smoe_route_noalloc(const smoe_config_t* c, const smoe_bf16_t* x, int64_t T,
                                            const float* w_router, const float* bias, int32_t* topk_idx,
                                            float* topk_w, float* logits_opt, void* stream) {
    // the same argument checks as smoe_route, before any launch
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
    const int sms = num_sms_current_device();
    const RouterPlan rp = router_plan(*c, T, sms, /*allow_tc=*/false);
    if (rp.scratch_bytes > (size_t)SMOE_NOALLOC_SCRATCH_BYTES) return SMOE_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (cudaGetSymbolAddress(&scratch, g_noalloc_scratch) != cudaSuccess || scratch == nullptr) return SMOE_ERR_CUDA;
    // Every element of the partial-logit area the kernels read is written first in the same
    // call, so nothing needs clearing.
    const cudaError_t e = launch_route(*c, x, T, w_router, bias, topk_idx, topk_w, logits_opt,
                                       static_cast<float*>(scratch), nullptr, sms, static_cast<cudaStream_t>(stream),
                                       /*allow_tc=*/false);
    return e == cudaSuccess ? SMOE_OK : SMOE_ERR_CUDA;
}
