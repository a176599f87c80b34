// e4m3 (FP8) experts: weight packing with per-row scales and per-row activation quantisation.
//
// Source: the Step 3.5 Flash summary (paperlayer.ai) fits the model into a 128 GB workstation
// memory budget, which calls for low-precision experts without naming a format. Quantiser (the
// same as the test oracle's, stated in include/stepmoe.h): each row of a matrix (a weight row =
// one output feature, an activation row = one token) gets s = max|row| / 448 in fp32 (1 for an
// all-zero row) and the codes e4m3(a / s), the division in IEEE fp32 and the conversion rounding
// to nearest even with saturation at +-448. The GEMM multiplies codes on the tensor cores
// (kind::f8f6f4) and scales the fp32 accumulator by s_w(feature) * s_a(token).
//
// Packed layout (tile-major like the bf16 experts, 128 e4m3 codes = 128 bytes per tile row):
//   gate/up codes [(E+1)][I/128][H/128][256][128]  tile (g, mb, kb): 128 gate rows of features
//                                                   128 mb .. +127, then the matching 128 up rows
//   down codes    [(E+1)][H/128][I/128][128][128]
//   gate/up scales [(E+1)][2][I] fp32 (gate rows, then up rows), down scales [(E+1)][H] fp32.
#include "common.cuh"
#include "internal.h"
#include "quant.cuh"

namespace smoe {

namespace {

__global__ void __launch_bounds__(256) quantize_rows_kernel(const uint16_t* __restrict__ a, int64_t rows, int cols,
                                                            uint8_t* __restrict__ q, float* __restrict__ scale) {
    const int lane = threadIdx.x & 31;
    pdl_wait();
    pdl_launch_dependents();
    for (int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); r < rows; r += (int64_t)gridDim.x * 8) {
        uint2* dst = reinterpret_cast<uint2*>(q + (size_t)r * cols);
        const float sc = quantize_row_warp(a + (size_t)r * cols, cols, [&](int v, uint2 c) { dst[v] = c; });
        if (lane == 0) scale[r] = sc;
    }
}

// One warp per weight row. gate/up row (g, f, up): tile block bi = g * (I/128) + f / 128, tile
// row (f % 128) + 128 * up; down row (g, f): bi = g * (H/128) + f / 128, tile row f % 128.
__global__ void __launch_bounds__(256) pack_fp8_kernel(const uint16_t* __restrict__ wg, const uint16_t* __restrict__ wu,
                                                       const uint16_t* __restrict__ wd, const uint16_t* __restrict__ sg,
                                                       const uint16_t* __restrict__ su, const uint16_t* __restrict__ sd,
                                                       int E, int I, int H, uint8_t* __restrict__ gu_q,
                                                       uint8_t* __restrict__ dn_q, float* __restrict__ gu_s,
                                                       float* __restrict__ dn_s) {
    const int lane = threadIdx.x & 31;
    const int64_t n_gu = (int64_t)(E + 1) * 2 * I, n_dn = (int64_t)(E + 1) * H;
    for (int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); r < n_gu + n_dn; r += (int64_t)gridDim.x * 8) {
        if (r < n_gu) {
            const int g = (int)(r / (2 * I));
            const int rr = (int)(r % (2 * I));
            const bool up = rr >= I;
            const int f = up ? rr - I : rr;
            const uint16_t* src = (g < E) ? ((up ? wu : wg) + ((size_t)g * I + f) * H) : ((up ? su : sg) + (size_t)f * H);
            const size_t bi = (size_t)g * (I / 128) + f / 128;
            const int trow = (f % 128) + (up ? 128 : 0);
            const float sc = quantize_row_warp(src, H, [&](int v, uint2 c) {
                const int k = v * 8;   // K element of this chunk
                const size_t tile = bi * (H / 128) + k / 128;
                *reinterpret_cast<uint2*>(gu_q + (tile * 256 + trow) * 128 + (k % 128)) = c;
            });
            if (lane == 0) gu_s[((size_t)g * 2 + (up ? 1 : 0)) * I + f] = sc;
        } else {
            const int64_t rd = r - n_gu;
            const int g = (int)(rd / H);
            const int f = (int)(rd % H);
            const uint16_t* src = (g < E) ? (wd + ((size_t)g * H + f) * I) : (sd + (size_t)f * I);
            const size_t bi = (size_t)g * (H / 128) + f / 128;
            const int trow = f % 128;
            const float sc = quantize_row_warp(src, I, [&](int v, uint2 c) {
                const int k = v * 8;
                const size_t tile = bi * (I / 128) + k / 128;
                *reinterpret_cast<uint2*>(dn_q + (tile * 128 + trow) * 128 + (k % 128)) = c;
            });
            if (lane == 0) dn_s[(size_t)g * H + f] = sc;
        }
    }
}

}  // namespace

Fp8Layout fp8_layout(const smoe_config_t& c) {
    Fp8Layout L;
    const size_t E1 = (size_t)c.n_experts + 1, H = c.hidden, I = c.inter;
    size_t o = 0;
    L.gateup = o;       o += align_up(E1 * 2 * I * H);
    L.down = o;         o += align_up(E1 * H * I);
    L.gateup_scale = o; o += align_up(E1 * 2 * I * 4);
    L.down_scale = o;   o += align_up(E1 * H * 4);
    L.total = o;
    return L;
}

cudaError_t launch_pack_fp8(const smoe_config_t& c, const uint16_t* wg, const uint16_t* wu, const uint16_t* wd,
                            const uint16_t* sg, const uint16_t* su, const uint16_t* sd, void* packed, cudaStream_t s) {
    const Fp8Layout L = fp8_layout(c);
    uint8_t* b = static_cast<uint8_t*>(packed);
    {
        LaunchTimer lt(K_PACK_FP8, s);
        pack_fp8_kernel<<<148 * 8, 256, 0, s>>>(wg, wu, wd, sg, su, sd, c.n_experts, c.inter, c.hidden, b + L.gateup,
                                                b + L.down, reinterpret_cast<float*>(b + L.gateup_scale),
                                                reinterpret_cast<float*>(b + L.down_scale));
    }
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) launches_add(1);
    return e;
}

cudaError_t launch_quantize_rows(const uint16_t* a, int64_t rows, int cols, uint8_t* q, float* scale, KernelId id,
                                 cudaStream_t s) {
    int64_t blocks = (rows + 7) / 8;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    cudaError_t e;
    {
        LaunchTimer lt(id, s);
        e = launch_pdl(quantize_rows_kernel, dim3((unsigned)blocks), dim3(256), 0, s, a, rows, cols, q, scale);
    }
    if (e == cudaSuccess) launches_add(1);
    return e;
}

}  // namespace smoe
