// Combine: out[t] = y[T*k + t] + sum_j w[t, j] * y[perm_row[t*k + j]].
// Source: every token's layer output is its shared-expert output plus the weighted outputs
// of its 8 routed experts (Step 3.5 Flash summary, hyper.ai, section "方法"; weights from the
// router, model card fields norm_expert_weight and moe_router_scaling_factor).
//
// One CTA per token; each thread owns 8 consecutive features (one 16-byte vector per row).
// Accumulation is fp32 in slot order j = 0..k-1, the shared row is added last, and the sum is
// rounded once to bf16. Rows outside [0, T*k) are skipped and set SMOE_ERR_DEVICE.
// With NORMS (smoe_forward_diag) the kernel also writes ||y[r]||_2 of each routed row it
// reads, the expert-output norm behind the per-expert monitoring of the Step 3.5 Flash summary
// (paperlayer.ai, §4.1.2-§4.1.3: per-expert activation norms, their max- and min-to-median
// ratios); the sum of squares is reduced in a fixed order, so the norms are deterministic.
#include "common.cuh"
#include "internal.h"

namespace smoe {

namespace {

constexpr int kMaxK = 32;

__device__ __forceinline__ void fma8(float (&acc)[8], float w, const uint4 v) {
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[2 * i] = fmaf(w, __uint_as_float(u[i] << 16), acc[2 * i]);
        acc[2 * i + 1] = fmaf(w, __uint_as_float(u[i] & 0xFFFF0000u), acc[2 * i + 1]);
    }
}

__device__ __forceinline__ float sumsq8(const uint4 v) {
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float a = __uint_as_float(u[i] << 16), b = __uint_as_float(u[i] & 0xFFFF0000u);
        s = fmaf(a, a, s);
        s = fmaf(b, b, s);
    }
    return s;
}

template <bool NORMS>
__global__ void __launch_bounds__(256, 3) combine_kernel(const uint16_t* __restrict__ y,
                                                      const int32_t* __restrict__ perm_row,
                                                      const float* __restrict__ topk_w, int T, int k, int H,
                                                      uint16_t* __restrict__ out, int32_t* err,
                                                      float* __restrict__ row_norm) {
    __shared__ int32_t rows[kMaxK];
    __shared__ float ws[kMaxK];
    __shared__ float red[NORMS ? 8 * 8 : 1];   // [warp][slot] partial sums of squares
    float sq[8];                               // NORMS, k <= 8: this thread's sums of squares per slot
    pdl_wait();
    pdl_launch_dependents();
#pragma unroll
    for (int j = 0; j < 8; ++j) sq[j] = 0.f;
    const int t = blockIdx.x;
    const int64_t nrouted = (int64_t)T * k;
    if (threadIdx.x < k) {
        int32_t r = perm_row[(size_t)t * k + threadIdx.x];
        if (r < 0 || r >= nrouted) {
            record_error(err, SMOE_ERR_DEVICE);
            r = -1;
        }
        rows[threadIdx.x] = r;
        ws[threadIdx.x] = topk_w[(size_t)t * k + threadIdx.x];
    }
    __syncthreads();
    const int vec = H / 8;
    const uint4* y4 = reinterpret_cast<const uint4*>(y);
    for (int c = threadIdx.x; c < vec; c += blockDim.x) {
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.f;
        const uint4 shared_row = y4[(size_t)(nrouted + t) * vec + c];
        if (k <= 8) {
            // all rows' vectors in flight first, then the FMAs in slot order
            uint4 v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (j < k && rows[j] >= 0) v[j] = y4[(size_t)rows[j] * vec + c];
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (j < k && rows[j] >= 0) {
                    fma8(acc, ws[j], v[j]);
                    if constexpr (NORMS) sq[j] += sumsq8(v[j]);
                }
        } else {
            for (int j = 0; j < k; ++j) {
                const int r = rows[j];
                if (r >= 0) fma8(acc, ws[j], y4[(size_t)r * vec + c]);
            }
        }
        fma8(acc, 1.0f, shared_row);
        uint4 o;
        uint32_t* ou = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            ou[i] = pack_bf16x2(acc[2 * i], acc[2 * i + 1]);
        reinterpret_cast<uint4*>(out)[(size_t)t * vec + c] = o;
    }
    if constexpr (NORMS) {
        // per slot: a warp butterfly, then the warps' partials in warp order (blockDim.x <= 256)
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
        if (k <= 8) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float v = sq[j];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
                if (lane == 0) red[warp * 8 + j] = v;
            }
            __syncthreads();
            if (threadIdx.x < k && rows[threadIdx.x] >= 0) {
                float tot = 0.f;
                for (int w = 0; w < nw; ++w) tot += red[w * 8 + threadIdx.x];
                row_norm[rows[threadIdx.x]] = sqrtf(tot);
            }
        } else {
            // k > 8: one slot at a time, re-reading its row (just loaded, so from L2)
            for (int j = 0; j < k; ++j) {
                const int r = rows[j];
                float v = 0.f;
                if (r >= 0)
                    for (int c = threadIdx.x; c < vec; c += blockDim.x) v += sumsq8(y4[(size_t)r * vec + c]);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
                __syncthreads();
                if (lane == 0) red[warp] = v;
                __syncthreads();
                if (threadIdx.x == 0 && r >= 0) {
                    float tot = 0.f;
                    for (int w = 0; w < nw; ++w) tot += red[w];
                    row_norm[r] = sqrtf(tot);
                }
            }
        }
    }
}

}  // namespace

cudaError_t launch_combine(const smoe_config_t& c, const uint16_t* y, const int32_t* perm_row, const float* topk_w,
                           int64_t T, uint16_t* out, int32_t* err, cudaStream_t s, float* row_norm_opt) {
    const int threads = c.hidden / 8 >= 256 ? 256 : 128;
    cudaError_t e;
    {
        LaunchTimer lt(K_COMBINE, s);
        if (row_norm_opt != nullptr)
            e = launch_pdl(combine_kernel<true>, dim3((unsigned)T), dim3(threads), 0, s, y, perm_row, topk_w, (int)T,
                           c.top_k, c.hidden, out, err, row_norm_opt);
        else
            e = launch_pdl(combine_kernel<false>, dim3((unsigned)T), dim3(threads), 0, s, y, perm_row, topk_w, (int)T,
                           c.top_k, c.hidden, out, err, (float*)nullptr);
    }
    if (e == cudaSuccess) launches_add(1);
    return e;
}

}  // namespace smoe
