// e4m3 row quantisation shared by the x quantiser (inside the router's top-k kernel), the
// standalone row quantiser and the weight packer: one warp per row, s = max|row| / 448 (1 for an
// all-zero row), codes e4m3(a / s) with the division in IEEE fp32, rounding to nearest even with
// saturation (the quantiser stated in include/stepmoe.h).
#pragma once

#include "common.cuh"

namespace smoe {

constexpr float kE4m3Max = 448.0f;

__device__ __forceinline__ float warp_absmax(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, off));
    return v;
}

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// One warp quantises one row of `cols` bf16 values (cols % 256 == 0 not required; cols % 8 == 0):
// returns the scale; writes the codes through put(k8, uint2 of 8 codes) for 8-element chunk k8.
template <typename Put>
__device__ __forceinline__ float quantize_row_warp(const uint16_t* __restrict__ row, int cols, Put put) {
    const int lane = threadIdx.x & 31;
    const uint4* r4 = reinterpret_cast<const uint4*>(row);
    const int nv = cols / 8;
    float amax = 0.f;
    for (int v = lane; v < nv; v += 32) {
        const uint4 q = r4[v];
        const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(u[i])), fabsf(bf16_hi(u[i]))));
    }
    amax = warp_absmax(amax);
    const float sc = amax > 0.f ? amax / kE4m3Max : 1.0f;   // IEEE division
    for (int v = lane; v < nv; v += 32) {
        const uint4 q = r4[v];
        const uint32_t u[4] = {q.x, q.y, q.z, q.w};
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t c0 = float_to_e4m3(bf16_lo(u[i]) / sc), c1 = float_to_e4m3(bf16_hi(u[i]) / sc);
            const uint32_t pair = c0 | (c1 << 8);
            if (i < 2) lo |= pair << (16 * i); else hi |= pair << (16 * (i - 2));
        }
        put(v, make_uint2(lo, hi));
    }
    return sc;
}

}  // namespace smoe
