// Weight packing for the expert GEMMs (a one-time layout transform, not part of a step).
// Tile-major: every weight tile one TMA load brings into shared memory (R rows x 64 K columns,
// 128-byte rows) is one contiguous block in HBM, so each load streams whole DRAM pages.
//   gate/up: [(E+1)][I/128][H/64][256][64] — tile (g, mb, kb): rows 0-127 the gate rows of
//            features 128 mb .. 128 mb + 127, rows 128-255 the matching up rows, columns
//            64 kb .. 64 kb + 63 of K = H; one 256-row box feeds both MMAs;
//   down:    [(E+1)][H/128][I/64][128][64]  — tile (g, mb, kb): rows 128 mb .. + 127 of W_d,
//            columns 64 kb .. + 63 of K = I.
// Group E is the shared expert (Step 3.5 Flash summary, hyper.ai, section "方法": one shared
// expert beside the routed ones; model card field share_expert_dim 1280).
#include "common.cuh"
#include "internal.h"

namespace smoe {

namespace {

// One thread per 16-byte chunk of a destination tile row (8 chunks = the row's 64 elements).
// Destination tile row tr = ((bi * KT + kb) * R + r) with bi = g * MB + mb; the source row of
// (g, mb, r) comes from src_row(), its columns 64 kb .. 64 kb + 63.
template <typename SrcRow>
__device__ __forceinline__ void pack_tiles(int64_t ntr, int R, int KT, int MB, int K, uint16_t* __restrict__ dst,
                                           SrcRow src_row) {
    const int64_t nchunks = ntr * 8;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nchunks; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t tr = i >> 3;
        const int ch = (int)(i & 7);
        const int r = (int)(tr % R);
        const int64_t tile = tr / R;
        const int kb = (int)(tile % KT);
        const int64_t bi = tile / KT;
        const int g = (int)(bi / MB), mb = (int)(bi % MB);
        const uint16_t* src = src_row(g, mb, r);
        reinterpret_cast<uint4*>(dst)[i] = *reinterpret_cast<const uint4*>(src + (size_t)kb * 64 + ch * 8);
    }
    (void)K;
}

__global__ void __launch_bounds__(256) pack_gateup_kernel(const uint16_t* __restrict__ wg,
                                                          const uint16_t* __restrict__ wu,
                                                          const uint16_t* __restrict__ sg,
                                                          const uint16_t* __restrict__ su, int E, int I, int H,
                                                          uint16_t* __restrict__ dst) {
    const int MB = I / 128, KT = H / 64;
    const int64_t ntr = (int64_t)(E + 1) * MB * KT * 256;
    pack_tiles(ntr, 256, KT, MB, H, dst, [&](int g, int mb, int r) {
        const int feat = mb * 128 + (r & 127);
        const bool up = r >= 128;
        return (g < E) ? ((up ? wu : wg) + ((size_t)g * I + feat) * H) : ((up ? su : sg) + (size_t)feat * H);
    });
}

__global__ void __launch_bounds__(256) pack_down_kernel(const uint16_t* __restrict__ wd,
                                                        const uint16_t* __restrict__ sd, int E, int I, int H,
                                                        uint16_t* __restrict__ dst) {
    const int MB = H / 128, KT = I / 64;
    const int64_t ntr = (int64_t)(E + 1) * MB * KT * 128;
    pack_tiles(ntr, 128, KT, MB, I, dst, [&](int g, int mb, int r) {
        const int row = mb * 128 + r;
        return (g < E) ? (wd + ((size_t)g * H + row) * I) : (sd + (size_t)row * I);
    });
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
