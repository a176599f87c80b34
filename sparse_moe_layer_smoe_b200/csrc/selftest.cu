// Self-test of the bounded mbarrier wait that every GEMM role uses (failure detection without a
// GPU fault): one thread initialises an mbarrier that nothing will ever arrive at and waits on it
// through the same routine with a short limit. The wait gives up, records SMOE_ERR_TIMEOUT in
// the workspace's error word and returns; the kernel exits normally and the context stays
// usable. Nothing here faults, traps or spins without a limit.
#include "common.cuh"
#include "internal.h"

namespace smoe {

namespace {

__global__ void wait_timeout_selftest_kernel(int32_t* err, uint64_t limit_ns, uint64_t* elapsed_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x != 0) return;
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
    const uint64_t t0 = globaltimer_ns();
    // parity 0: the barrier's first phase, which completes only after one arrival (none comes)
    const bool ok = mbar_wait_for(smem_u32(&bar), 0u, err, &abort_flag, false, limit_ns);
    if (elapsed_ns != nullptr) *elapsed_ns = globaltimer_ns() - t0;
    if (ok) record_error(err, SMOE_ERR_DEVICE);   // cannot happen: nothing arrived
}

// The gate/up epilogue's SiLU(g) * u (silu_mul, as the GEMM epilogue computes it), one element
// per thread.
__global__ void swiglu_selftest_kernel(const float* g, const float* u, int64_t n, float* out) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) out[i] = silu_mul(g[i], u[i]);
}

}  // namespace

cudaError_t launch_swiglu_selftest(const float* g, const float* u, int64_t n, float* out, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    swiglu_selftest_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(g, u, n, out);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) launches_add(1);
    return e;
}

cudaError_t launch_wait_selftest(int32_t* err, uint64_t limit_ns, uint64_t* elapsed_ns, cudaStream_t s) {
    wait_timeout_selftest_kernel<<<1, 32, 0, s>>>(err, limit_ns, elapsed_ns);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) launches_add(1);
    return e;
}

}  // namespace smoe
