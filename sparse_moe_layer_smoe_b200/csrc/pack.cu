// Weight packing for the expert GEMMs (a one-time layout transform, not part of a step).
//   gate/up block: [(E+1)][I/128][2][128][H]  — per 128-feature block, the 128 gate rows then
//                  the 128 matching up rows, so one 256-row TMA box feeds both MMAs;
//   down block:    [(E+1)][H][I]              — routed experts then the shared expert.
// Group E is the shared expert (Step 3.5 Flash summary, hyper.ai, section "方法": one shared
// expert beside the routed ones; model card field share_expert_dim 1280).
#include "common.cuh"
#include "internal.h"

namespace smoe {

namespace {

// One warp per destination row; rows are copied with 16-byte vectors.
__global__ void __launch_bounds__(256) pack_gateup_kernel(const uint16_t* __restrict__ wg,
                                                          const uint16_t* __restrict__ wu,
                                                          const uint16_t* __restrict__ sg,
                                                          const uint16_t* __restrict__ su, int E, int I, int H,
                                                          uint16_t* __restrict__ dst) {
    const int64_t nrows = (int64_t)(E + 1) * 2 * I;
    const int lane = threadIdx.x & 31;
    const int vec = H / 8;
    for (int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); r < nrows; r += (int64_t)gridDim.x * 8) {
        const int g = (int)(r / (2 * I));
        const int rr = (int)(r % (2 * I));
        const int mb = rr / 256, w = rr % 256;
        const int feat = mb * 128 + (w & 127);
        const bool up = w >= 128;
        const uint16_t* src = (g < E) ? ((up ? wu : wg) + ((size_t)g * I + feat) * H) : ((up ? su : sg) + (size_t)feat * H);
        const uint4* s4 = reinterpret_cast<const uint4*>(src);
        uint4* d4 = reinterpret_cast<uint4*>(dst + (size_t)r * H);
        for (int c = lane; c < vec; c += 32) d4[c] = s4[c];
    }
}

__global__ void __launch_bounds__(256) pack_down_kernel(const uint16_t* __restrict__ wd,
                                                        const uint16_t* __restrict__ sd, int E, int I, int H,
                                                        uint16_t* __restrict__ dst) {
    const int64_t nrows = (int64_t)(E + 1) * H;
    const int lane = threadIdx.x & 31;
    const int vec = I / 8;
    for (int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); r < nrows; r += (int64_t)gridDim.x * 8) {
        const int g = (int)(r / H);
        const uint16_t* src = (g < E) ? (wd + (size_t)r * I) : (sd + (size_t)(r - (int64_t)E * H) * I);
        const uint4* s4 = reinterpret_cast<const uint4*>(src);
        uint4* d4 = reinterpret_cast<uint4*>(dst + (size_t)r * I);
        for (int c = lane; c < vec; c += 32) d4[c] = s4[c];
    }
}

}  // namespace

cudaError_t launch_pack(const smoe_config_t& c, const uint16_t* wg, const uint16_t* wu, const uint16_t* wd,
                        const uint16_t* sg, const uint16_t* su, const uint16_t* sd, void* packed, cudaStream_t s) {
    uint16_t* gu = static_cast<uint16_t*>(packed);
    uint16_t* dn = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(packed) + packed_gateup_bytes(c));
    const int blocks = 148 * 8;
    {
        LaunchTimer lt(K_PACK_GATEUP, s);
        pack_gateup_kernel<<<blocks, 256, 0, s>>>(wg, wu, sg, su, c.n_experts, c.inter, c.hidden, gu);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    {
        LaunchTimer lt(K_PACK_DOWN, s);
        pack_down_kernel<<<blocks, 256, 0, s>>>(wd, sd, c.n_experts, c.inter, c.hidden, dn);
    }
    e = cudaGetLastError();
    if (e == cudaSuccess) launches_add(2);
    return e;
}

}  // namespace smoe
