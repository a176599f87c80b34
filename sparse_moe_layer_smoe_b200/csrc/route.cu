// Router: fp32 logits L = x W_r^T (x bf16, upcast exactly), sigmoid scores s, biased scores
// s + bias for selection, top-k, weights route_scale * s_j / sum s_j.
//
// Source: Step-3.5-Flash model card (llm-atlas), raw config fields need_fp32_gate,
// moe_router_activation sigmoid, use_moe_router_bias, moe_top_k 8, norm_expert_weight,
// moe_router_scaling_factor 3; the bias steers selection only (Step 3.5 Flash summary,
// paperlayer.ai, §4.1.2: loss-free bias adjustment as the balancing device).
//
// Logits, small T (router_logits_kernel): a register-tiled fp32 SGEMM on the CUDA cores. Each
// CTA owns TM tokens x TE experts over one K range; K is split only when T is small, so the
// 4.7 MB of W_r is spread over all SMs at decode sizes. Partial sums go to the workspace.
// Logits, T >= 512 (router_split_kernel + the grouped tensor-core GEMM in router mode): W_r is
// split exactly into three bf16 pieces, so x W_r^T = x W_hi^T + x W_mid^T + x W_lo^T with
// every product exact, accumulated in fp32 in TMEM (19 GFLOP of fp32 at T = 8192 become
// 58 GFLOP of bf16 on the tensor cores); each piece's K range may be cut into 2 or 4 parts so
// that small batches still cover the SMs, one partial per part.
// Kernel 2 (router_topk_kernel): one warp per token adds the K-split partials in a fixed
// order (deterministic), applies sigmoid and bias, and selects top-k in k rounds of a warp
// argmax over 64-bit keys (biased score, then logit; warp max reductions), the smaller expert
// index winning an exact tie; then normalises.
#include <float.h>

#include "common.cuh"
#include "internal.h"
#include "quant.cuh"

namespace smoe {

namespace {

template <int TM, int TE, int RM, int RE, int KC_>
struct RouterTile {
    static constexpr int TX = TE / RE;          // threads along experts
    static constexpr int TY = TM / RM;          // threads along tokens
    static constexpr int THREADS = TX * TY;
    static constexpr int KC = KC_;              // K elements per stage
    static constexpr int XCHUNKS = TM * KC / 8; // 16-byte chunks of x per stage
    static constexpr int WCHUNKS = TE * KC / 4; // 16-byte chunks of W_r per stage
    static constexpr int XPT = (XCHUNKS + THREADS - 1) / THREADS;
    static constexpr int WPT = (WCHUNKS + THREADS - 1) / THREADS;
};

template <int TM, int TE, int RM, int RE, int KC_>
__global__ void __launch_bounds__(RouterTile<TM, TE, RM, RE, KC_>::THREADS)
router_logits_kernel(const uint16_t* __restrict__ x, const float* __restrict__ wr, float* __restrict__ part,
                     int T, int E, int H, int k_len) {
    using P = RouterTile<TM, TE, RM, RE, KC_>;
    constexpr int KC = P::KC;
    pdl_wait();
    pdl_launch_dependents();
    // two stages of x [KC][TM+1] and W_r [KC][TE+1]; +1 padding: the transposing stores below
    // hit 32 distinct banks
    extern __shared__ float rsm[];
    float (*xs)[KC][TM + 1] = reinterpret_cast<float (*)[KC][TM + 1]>(rsm);
    float (*ws)[KC][TE + 1] = reinterpret_cast<float (*)[KC][TE + 1]>(rsm + 2 * KC * (TM + 1));

    const int tid = threadIdx.x;
    const int tx = tid % P::TX, ty = tid / P::TX;
    const int t0 = blockIdx.x * TM, e0 = blockIdx.y * TE;
    const int kbeg = blockIdx.z * k_len;
    const int nchunks = k_len / KC;

    uint4 xr[P::XPT];
    float4 wrg[P::WPT];

    auto gload = [&](int kc) {
        const int kb = kbeg + kc * KC;
#pragma unroll
        for (int i = 0; i < P::XPT; ++i) {
            const int c = tid + i * P::THREADS;
            xr[i] = make_uint4(0, 0, 0, 0);
            if (c < P::XCHUNKS) {
                const int m = c / (KC / 8), q = c % (KC / 8);
                const int t = t0 + m;
                if (t < T) xr[i] = *reinterpret_cast<const uint4*>(x + (size_t)t * H + kb + q * 8);
            }
        }
#pragma unroll
        for (int i = 0; i < P::WPT; ++i) {
            const int c = tid + i * P::THREADS;
            wrg[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (c < P::WCHUNKS) {
                const int n = c / (KC / 4), q = c % (KC / 4);
                const int e = e0 + n;
                if (e < E) wrg[i] = *reinterpret_cast<const float4*>(wr + (size_t)e * H + kb + q * 4);
            }
        }
    };
    auto sstore = [&](int buf) {
#pragma unroll
        for (int i = 0; i < P::XPT; ++i) {
            const int c = tid + i * P::THREADS;
            if (c < P::XCHUNKS) {
                const int m = c / (KC / 8), q = c % (KC / 8);
                const uint32_t w4[4] = {xr[i].x, xr[i].y, xr[i].z, xr[i].w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    xs[buf][q * 8 + 2 * h][m] = __uint_as_float(w4[h] << 16);
                    xs[buf][q * 8 + 2 * h + 1][m] = __uint_as_float(w4[h] & 0xFFFF0000u);
                }
            }
        }
#pragma unroll
        for (int i = 0; i < P::WPT; ++i) {
            const int c = tid + i * P::THREADS;
            if (c < P::WCHUNKS) {
                const int n = c / (KC / 4), q = c % (KC / 4);
                ws[buf][q * 4 + 0][n] = wrg[i].x;
                ws[buf][q * 4 + 1][n] = wrg[i].y;
                ws[buf][q * 4 + 2][n] = wrg[i].z;
                ws[buf][q * 4 + 3][n] = wrg[i].w;
            }
        }
    };

    float acc[RM][RE];
#pragma unroll
    for (int i = 0; i < RM; ++i)
#pragma unroll
        for (int j = 0; j < RE; ++j) acc[i][j] = 0.f;

    gload(0);
    sstore(0);
    __syncthreads();
    for (int kc = 0; kc < nchunks; ++kc) {
        const int buf = kc & 1;
        if (kc + 1 < nchunks) gload(kc + 1);
#pragma unroll 8
        for (int kk = 0; kk < KC; ++kk) {
            float a[RM], b[RE];
#pragma unroll
            for (int i = 0; i < RM; ++i) a[i] = xs[buf][kk][ty * RM + i];
#pragma unroll
            for (int j = 0; j < RE; ++j) b[j] = ws[buf][kk][tx * RE + j];
#pragma unroll
            for (int i = 0; i < RM; ++i)
#pragma unroll
                for (int j = 0; j < RE; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        if (kc + 1 < nchunks) sstore(buf ^ 1);
        __syncthreads();
    }

    float* dst = part + (size_t)blockIdx.z * T * E;
#pragma unroll
    for (int i = 0; i < RM; ++i) {
        const int t = t0 + ty * RM + i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < RE; ++j) {
            const int e = e0 + tx * RE + j;
            if (e < E) dst[(size_t)t * E + e] = acc[i][j];
        }
    }
}

// Order-preserving map of a float to an unsigned key (a < b exactly when key(a) < key(b));
// -0 is folded into +0 first, as the float comparison treats them as equal.
__device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t u = __float_as_uint(f + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// QX: 0 = no x quantisation (bf16 layer); 1 = quantise x before the dependency wait (the router
// kernel before it is the CUDA-core one, beside which this grid's CTAs can already run);
// 2 = quantise x at the end (after a tensor-core router GEMM, which leaves no room to co-run,
// and where the first variant's extra registers cost occupancy).
template <int NPL, int QX>
__global__ void __launch_bounds__(256)
router_topk_kernel(const float* __restrict__ part, int splits, const float* __restrict__ bias, int T, int E, int k,
                   float scale, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                   float* __restrict__ logits_out, float* __restrict__ conf_out, const uint16_t* __restrict__ x,
                   int H, uint8_t* __restrict__ x_q, float* __restrict__ s_x) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (QX == 1 && t < T) {
        // e4m3 layer: this token's row of x quantised here, saving a launch. x does not come
        // from the router, so this runs before the wait, while the router kernel still works:
        // this grid only launches once the router kernel has passed its own wait, i.e. after
        // every kernel of the previous layer call (the last readers of x_q) has completed.
        uint2* dst = reinterpret_cast<uint2*>(x_q + (size_t)t * H);
        const float sc = quantize_row_warp(x + (size_t)t * H, H, [&](int v, uint2 c) { dst[v] = c; });
        if (lane == 0) s_x[t] = sc;
    }
    pdl_wait();
    pdl_launch_dependents();
    if (t >= T) return;

    // logits: the K-split partials added in split order 0, 1, 2, ... (the order is fixed, so the
    // result is deterministic); all loads of a group of G splits are issued before the first add
    constexpr int G = NPL <= 16 ? 4 : 2;
    const float* pt = part + (size_t)t * E + lane;
    const size_t stride = (size_t)T * E;
    float L[NPL], S[NPL], B[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        L[i] = 0.f;
        B[i] = (lane + 32 * i < E) ? bias[lane + 32 * i] : 0.f;
    }
    for (int s0 = 0; s0 < splits; s0 += G) {
        float v[G][NPL];
#pragma unroll
        for (int q = 0; q < G; ++q)
#pragma unroll
            for (int i = 0; i < NPL; ++i)
                v[q][i] = (s0 + q < splits && lane + 32 * i < E) ? pt[(size_t)(s0 + q) * stride + 32 * i] : 0.f;
#pragma unroll
        for (int q = 0; q < G; ++q)
#pragma unroll
            for (int i = 0; i < NPL; ++i)
                if (s0 + q < splits) L[i] += v[q][i];
    }
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int e = lane + 32 * i;
        S[i] = 0.f;
        if (e < E) {
            const float l = L[i];
            if (logits_out) logits_out[(size_t)t * E + e] = l;
            const float sg = 1.0f / (1.0f + expf(-l));
            S[i] = sg;
            const float bb = sg + B[i];
            B[i] = (bb != bb) ? -INFINITY : bb;
            if (l != l) L[i] = -FLT_MAX;
        }
    }

    // Selection order: larger biased score, then larger logit, then smaller expert index.
    // Each candidate carries the 64-bit key (key(b^), key(logit)); a taken or absent candidate
    // has key 0, below every real one (key(-inf) > 0), and k <= E leaves a real one each round.
    uint32_t kh[NPL], kl[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const bool live = lane + 32 * i < E;
        kh[i] = live ? order_key(B[i]) : 0u;
        kl[i] = live ? order_key(L[i]) : 0u;
    }
    float s_sel = 0.f;   // this lane's copy of the chosen score for slot j == lane
    int e_sel = 0;
    for (int j = 0; j < k; ++j) {
        // this lane's best: strict comparison in ascending i keeps the smaller index on a tie
        uint32_t bh = 0, bl = 0;
        int bi = 0;
#pragma unroll
        for (int i = 0; i < NPL; ++i)
            if (kh[i] > bh || (kh[i] == bh && kl[i] > bl)) {
                bh = kh[i];
                bl = kl[i];
                bi = i;
            }
        // warp-wide: the largest key, then the smallest index among the lanes holding it
        const uint32_t mh = __reduce_max_sync(0xFFFFFFFFu, bh);
        const uint32_t ml = __reduce_max_sync(0xFFFFFFFFu, bh == mh ? bl : 0u);
        const uint32_t ee = __reduce_min_sync(0xFFFFFFFFu, (bh == mh && bl == ml) ? (uint32_t)(lane + 32 * bi)
                                                                                   : 0xFFFFFFFFu);
        // the winning lane clears the winner's key; written as selects over every slot so the
        // arrays stay in registers (a store at a computed index would move them to local memory)
        const int wq = ((int)(ee & 31u) == lane) ? (int)(ee >> 5) : -1;
        float sw = 0.f;
#pragma unroll
        for (int q = 0; q < NPL; ++q) {
            const bool hit = q == wq;
            sw = hit ? S[q] : sw;
            kh[q] = hit ? 0u : kh[q];
            kl[q] = hit ? 0u : kl[q];
        }
        sw = __shfl_sync(0xFFFFFFFFu, sw, ee & 31u);
        if (lane == j) {
            s_sel = sw;
            e_sel = (int)ee;
        }
    }
    // sum of the selected unbiased scores in slot order j = 0..k-1
    float sum = 0.f;
    for (int j = 0; j < k; ++j) sum += __shfl_sync(0xFFFFFFFFu, s_sel, j);
    if (lane < k) {
        topk_idx[(size_t)t * k + lane] = e_sel;
        topk_w[(size_t)t * k + lane] = scale * (s_sel / sum);
    }
    if (conf_out != nullptr && lane == 0) conf_out[t] = sum / (float)k;   // routing confidence
    if (QX == 2) {
        uint2* dst = reinterpret_cast<uint2*>(x_q + (size_t)t * H);
        const float sc = quantize_row_warp(x + (size_t)t * H, H, [&](int v, uint2 c) { dst[v] = c; });
        if (lane == 0) s_x[t] = sc;
    }
}

// W_split[e][p*H + h] = piece p (0 = hi, 1 = mid, 2 = lo) of W_r[e][h]: hi = bf16(w),
// mid = bf16(w - hi), lo = bf16(w - hi - mid), each difference exact in fp32, so
// hi + mid + lo reproduces w to about 2^-24 relative and every product with a bf16 x is exact
// in fp32. Rows e >= E (padding up to a multiple of 128) are zero.
// Grid: (H/4/256 rounded up, e_pad); thread = 4 consecutive elements of row blockIdx.y.
__global__ void __launch_bounds__(256) router_split_kernel(const float* __restrict__ wr, int E, int H,
                                                           uint16_t* __restrict__ w_split) {
    pdl_wait();
    pdl_launch_dependents();
    const int e = blockIdx.y;
    const int c = blockIdx.x * 256 + threadIdx.x;   // 4-element column group
    if (4 * c >= H) return;
    float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
    if (e < E) w = *reinterpret_cast<const float4*>(wr + (size_t)e * H + 4 * c);
    const float v[4] = {w.x, w.y, w.z, w.w};
    uint32_t pc[3][2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        uint32_t h2 = 0, m2 = 0, l2 = 0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float f = v[2 * q + h];
            const uint16_t p0 = float_to_bf16_bits(f);
            const float r1 = f - bf16_bits_to_float(p0);
            const uint16_t p1 = float_to_bf16_bits(r1);
            const uint16_t p2 = float_to_bf16_bits(r1 - bf16_bits_to_float(p1));
            h2 |= (uint32_t)p0 << (16 * h);
            m2 |= (uint32_t)p1 << (16 * h);
            l2 |= (uint32_t)p2 << (16 * h);
        }
        pc[0][q] = h2;
        pc[1][q] = m2;
        pc[2][q] = l2;
    }
    uint16_t* row = w_split + (size_t)e * 3 * H + 4 * c;
#pragma unroll
    for (int piece = 0; piece < 3; ++piece)
        *reinterpret_cast<uint2*>(row + (size_t)piece * H) = make_uint2(pc[piece][0], pc[piece][1]);
}

template <int TM, int TE, int RM, int RE, int KC>
cudaError_t launch_logits(const uint16_t* x, int64_t T, const float* wr, int E, int H, int splits, float* part,
                          cudaStream_t s) {
    using P = RouterTile<TM, TE, RM, RE, KC>;
    dim3 grid((unsigned)((T + TM - 1) / TM), (unsigned)((E + TE - 1) / TE), (unsigned)splits);
    const int smem = (int)(2 * KC * (TM + 1 + TE + 1) * sizeof(float));
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(router_logits_kernel<TM, TE, RM, RE, KC>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
    }
    {
        LaunchTimer lt(K_ROUTER_LOGITS, s);
        return launch_pdl(router_logits_kernel<TM, TE, RM, RE, KC>, grid, dim3(P::THREADS), smem, s, x, wr, part,
                          (int)T, E, H, H / splits);
    }
}

template <int NPL>
cudaError_t launch_topk(const float* part, int splits, const float* bias, int64_t T, int E, int k, float scale,
                        int32_t* idx, float* w, float* logits, float* conf, const uint16_t* x, int H, uint8_t* x_q,
                        float* s_x, bool after_tc_router, cudaStream_t s) {
    const int warps = 8;
    const dim3 grid((unsigned)((T + warps - 1) / warps)), block(warps * 32);
    {
        LaunchTimer lt(K_ROUTER_TOPK, s);
        if (x_q == nullptr)
            return launch_pdl(router_topk_kernel<NPL, 0>, grid, block, 0, s, part, splits, bias, (int)T, E, k, scale,
                              idx, w, logits, conf, x, H, x_q, s_x);
        if (!after_tc_router)
            return launch_pdl(router_topk_kernel<NPL, 1>, grid, block, 0, s, part, splits, bias, (int)T, E, k, scale,
                              idx, w, logits, conf, x, H, x_q, s_x);
        return launch_pdl(router_topk_kernel<NPL, 2>, grid, block, 0, s, part, splits, bias, (int)T, E, k, scale, idx,
                          w, logits, conf, x, H, x_q, s_x);
    }
}

}  // namespace

// Tokens at which the router moves to the tensor cores (3-way bf16 split of W_r).
#ifndef SMOE_ROUTER_TC_MIN_T
#define SMOE_ROUTER_TC_MIN_T 512
#endif
constexpr int64_t kRouterTensorCoreMinT = SMOE_ROUTER_TC_MIN_T;
#ifndef SMOE_ROUTER_WIDE_TILE_MAX_T
#define SMOE_ROUTER_WIDE_TILE_MAX_T 64
#endif
// Batches up to this many tokens use the 64-token router tile.
constexpr int64_t kRouterWideTileMaxT = SMOE_ROUTER_WIDE_TILE_MAX_T;

RouterPlan router_plan(const smoe_config_t& c, int64_t T, int num_sms, bool allow_tc) {
    RouterPlan p{};
    const int E = c.n_experts;
    if (allow_tc && T >= kRouterTensorCoreMinT) {
        p.tc = true;
        p.e_pad = (E + 127) / 128 * 128;
        const int mb = p.e_pad / 128;
        p.nt = 256;
        const int64_t enough = (3 * (int64_t)num_sms) / 4;   // one round of units on 3/4 of the SMs
        while (p.nt > 64 && ((T + p.nt - 1) / p.nt) * mb * 3 < enough) p.nt /= 2;
        // K = the three bf16 pieces of W_r, each in m equal ranges: one partial per range,
        // summed in order by the top-k kernel (m grows until the units cover the SMs)
        int m = 1;
        while (m < 4 && c.hidden % (128 * m) == 0 && ((T + p.nt - 1) / p.nt) * mb * 3 * m < enough) m *= 2;
        p.splits = 3 * m;
        const size_t logit_b = ((size_t)p.splits * T * E * 4 + 255) / 256 * 256;
        p.scratch_bytes = logit_b + (size_t)p.e_pad * 3 * c.hidden * 2;
        return p;
    }
    if (T >= 512) {
        p.tm = 64;
        p.te = (E % 96 == 0) ? 96 : 64;
        p.kc = 32;
    } else if (T <= kRouterWideTileMaxT) {
        // every token of the batch in one tile: each W_r element is read by one CTA, and each
        // thread's 4 x 4 register tile takes two 16-byte shared loads per 16 FMAs
        p.tm = 64;
        p.te = 32;
        p.kc = 64;
        p.wide = true;
    } else {
        p.tm = 16;
        p.te = 32;
        p.kc = 128;   // few, long K slices: each CTA waits on 4 load rounds, not 16
    }
    const int64_t base = ((T + p.tm - 1) / p.tm) * ((E + p.te - 1) / p.te);
    const int chunks = c.hidden / p.kc;
    int splits = 1;
    while (splits * 2 <= 16 && chunks % (splits * 2) == 0 && base * splits * 2 <= 2 * (int64_t)num_sms) splits *= 2;
    p.splits = splits;
    p.scratch_bytes = (size_t)splits * T * E * 4;
    return p;
}

cudaError_t launch_route(const smoe_config_t& c, const uint16_t* x, int64_t T, const float* wr, const float* bias,
                         int32_t* topk_idx, float* topk_w, float* logits_opt, float* partials, int32_t* err,
                         int num_sms, cudaStream_t s, bool allow_tc, float* conf_opt, uint8_t* x_q_opt,
                         float* s_x_opt) {
    (void)err;
    const RouterPlan p = router_plan(c, T, num_sms, allow_tc);
    const int E = c.n_experts, H = c.hidden;
    cudaError_t e;
    int n = 2;
    if (p.tc) {
        const size_t logit_b = ((size_t)p.splits * T * E * 4 + 255) / 256 * 256;
        uint16_t* w_split = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(partials) + logit_b);
        {
            LaunchTimer lt(K_ROUTER_SPLIT, s);
            e = launch_pdl(router_split_kernel, dim3((unsigned)((H / 4 + 255) / 256), (unsigned)p.e_pad), dim3(256), 0,
                           s, wr, E, H, w_split);
        }
        if (e != cudaSuccess) return e;
        e = launch_router_gemm(x, T, H, w_split, p.e_pad, E, partials, p.nt, p.splits, num_sms, s);
        n = 3;
    } else if (p.wide) {
        e = launch_logits<64, 32, 4, 4, 64>(x, T, wr, E, H, p.splits, partials, s);
    } else if (p.tm == 64 && p.te == 96) {
        e = launch_logits<64, 96, 4, 6, 32>(x, T, wr, E, H, p.splits, partials, s);
    } else if (p.tm == 64) {
        e = launch_logits<64, 64, 4, 4, 32>(x, T, wr, E, H, p.splits, partials, s);
    } else {
        e = launch_logits<16, 32, 2, 2, 128>(x, T, wr, E, H, p.splits, partials, s);
    }
    if (e != cudaSuccess) return e;
    const int npl = (E + 31) / 32;
    if (npl <= 4)
        e = launch_topk<4>(partials, p.splits, bias, T, E, c.top_k, c.route_scale, topk_idx, topk_w, logits_opt, conf_opt, x, H, x_q_opt, s_x_opt, p.tc, s);
    else if (npl <= 9)
        e = launch_topk<9>(partials, p.splits, bias, T, E, c.top_k, c.route_scale, topk_idx, topk_w, logits_opt, conf_opt, x, H, x_q_opt, s_x_opt, p.tc, s);
    else if (npl <= 16)
        e = launch_topk<16>(partials, p.splits, bias, T, E, c.top_k, c.route_scale, topk_idx, topk_w, logits_opt, conf_opt, x, H, x_q_opt, s_x_opt, p.tc, s);
    else
        e = launch_topk<32>(partials, p.splits, bias, T, E, c.top_k, c.route_scale, topk_idx, topk_w, logits_opt, conf_opt, x, H, x_q_opt, s_x_opt, p.tc, s);
    if (e == cudaSuccess) launches_add(n);
    return e;
}

}  // namespace smoe
