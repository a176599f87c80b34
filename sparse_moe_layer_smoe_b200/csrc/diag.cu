// Layer monitoring outputs of smoe_forward_diag: per-expert token counts and expert-output norm
// statistics, per-token routing confidence (written by the top-k kernel) and a layer summary.
// Source: Step 3.5 Flash summary (paperlayer.ai): §4.1.2 (monitor per-expert activation norms;
// a falling minimum-to-median ratio warns of expert death), §4.1.3 (the maximum-to-median
// activation-norm ratio exposes localized activation blow-up while median norms stay flat),
// §5.2.1 (routing confidence as a proxy for MoE stability).
//
// One CTA of 1024 threads, after combine has written ||y[r]||_2 for every routed row r:
//   1. per expert, the count offsets[e+1] - offsets[e] and the mean and max of the norms of its
//      rows: a thread per expert when experts hold fewer than 32 rows on average, else a warp
//      per expert (lane-strided partial sums, then a butterfly); a fixed order either way;
//   2. each expert with tokens finds the rank of its mean among them (ties by expert index), so
//      the experts of rank (n-1)/2 and n/2 give the median, ranks 0 and n-1 the extremes;
//   3. block reductions in a fixed order give the rest of the summary.
// Every value is deterministic.
#include <float.h>

#include "common.cuh"
#include "internal.h"

namespace smoe {

namespace {

constexpr int kDiagThreads = 1024;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, off));
    return v;
}
__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = fminf(v, __shfl_xor_sync(0xFFFFFFFFu, v, off));
    return v;
}

__global__ void __launch_bounds__(kDiagThreads) diag_kernel(const float* __restrict__ row_norm,
                                                            const int32_t* __restrict__ offsets,
                                                            const float* __restrict__ conf, int E, int T, int k,
                                                            int32_t* __restrict__ count, float* __restrict__ norm_mean,
                                                            float* __restrict__ norm_max, float* __restrict__ summary,
                                                            int32_t* err) {
    __shared__ float s_mean[kDiagThreads], s_max[kDiagThreads];
    __shared__ int s_cnt[kDiagThreads], s_off[kDiagThreads + 1];
    __shared__ float s_red[32][5];
    __shared__ float s_rank[4];   // means of rank (n-1)/2, n/2, 0 and n-1
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int routed = T * k;
    pdl_wait();
    pdl_launch_dependents();
    for (int i = tid; i <= E; i += kDiagThreads) s_off[i] = offsets[i];
    __syncthreads();

    // 1. per expert: a thread per expert when experts hold few rows (decode), else a warp per
    //    expert; either way the partial sums are added in a fixed order
    auto store = [&](int e, int n, float sum, float mx) {
        const float mean = n > 0 ? sum / (float)n : 0.f;
        count[e] = n;
        norm_mean[e] = mean;
        norm_max[e] = mx;
        s_cnt[e] = n;
        s_mean[e] = mean;
        s_max[e] = mx;
    };
    auto bounds = [&](int e, int& o0, int& o1) {
        o0 = s_off[e];
        o1 = s_off[e + 1];
        if (o0 < 0 || o1 < o0 || o1 > routed) {
            record_error(err, SMOE_ERR_DEVICE);
            o0 = o1 = 0;
        }
    };
    if (routed < 32 * E) {
        for (int e = tid; e < E; e += kDiagThreads) {
            int o0, o1;
            bounds(e, o0, o1);
            float part[4] = {0.f, 0.f, 0.f, 0.f};
            float mx = 0.f;
            for (int r0 = o0; r0 < o1; r0 += 4) {
                float v[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) v[i] = (r0 + i < o1) ? row_norm[r0 + i] : 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    part[i] += v[i];
                    mx = fmaxf(mx, v[i]);
                }
            }
            store(e, o1 - o0, (part[0] + part[1]) + (part[2] + part[3]), mx);
        }
    } else {
        for (int e = warp; e < E; e += 32) {
            int o0, o1;
            bounds(e, o0, o1);
            // eight loads in flight per lane, eight partial sums added in a fixed order
            float part[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            float mx = 0.f;
            for (int r0 = o0 + lane; r0 < o1; r0 += 256) {
                float v[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = (r0 + 32 * i < o1) ? row_norm[r0 + 32 * i] : 0.f;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    part[i] += v[i];
                    mx = fmaxf(mx, v[i]);
                }
            }
            float sum = ((part[0] + part[1]) + (part[2] + part[3])) + ((part[4] + part[5]) + (part[6] + part[7]));
            sum = warp_sum(sum);
            mx = warp_max(mx);
            if (lane == 0) store(e, o1 - o0, sum, mx);
        }
    }
    __syncthreads();

    // 2. ranks among the experts with tokens (E <= kDiagThreads: one thread per expert)
    const int n_active = __syncthreads_count(tid < E && s_cnt[tid] > 0);
    if (tid < E && s_cnt[tid] > 0) {
        const float v = s_mean[tid];
        int rank = 0;
        for (int f = 0; f < E; ++f)
            if (s_cnt[f] > 0 && (s_mean[f] < v || (s_mean[f] == v && f < tid))) ++rank;
        if (rank == (n_active - 1) / 2) s_rank[0] = v;
        if (rank == n_active / 2) s_rank[1] = v;
        if (rank == 0) s_rank[2] = v;
        if (rank == n_active - 1) s_rank[3] = v;
    }
    __syncthreads();

    // 3. reductions: active experts, largest count, largest single norm; confidence mean and min
    float active = 0.f, cmax = 0.f, nmax = 0.f, csum = 0.f, cmin = INFINITY;
    for (int e = tid; e < E; e += kDiagThreads) {
        active += s_cnt[e] > 0 ? 1.f : 0.f;
        cmax = fmaxf(cmax, (float)s_cnt[e]);
        nmax = fmaxf(nmax, s_max[e]);
    }
    for (int t = tid; t < T; t += kDiagThreads) {
        csum += conf[t];
        cmin = fminf(cmin, conf[t]);
    }
    active = warp_sum(active);
    cmax = warp_max(cmax);
    nmax = warp_max(nmax);
    csum = warp_sum(csum);
    cmin = warp_min(cmin);
    if (lane == 0) {
        s_red[warp][0] = active;
        s_red[warp][1] = cmax;
        s_red[warp][2] = nmax;
        s_red[warp][3] = csum;
        s_red[warp][4] = cmin;
    }
    __syncthreads();
    if (tid == 0) {
        float a = 0.f, cm = 0.f, nm = 0.f, cs = 0.f, cn = INFINITY;
        for (int w = 0; w < 32; ++w) {
            a += s_red[w][0];
            cm = fmaxf(cm, s_red[w][1]);
            nm = fmaxf(nm, s_red[w][2]);
            cs += s_red[w][3];
            cn = fminf(cn, s_red[w][4]);
        }
        float med = 0.f, lo = 0.f, hi = 0.f;
        if (n_active > 0) {
            med = (n_active & 1) ? s_rank[1] : 0.5f * (s_rank[0] + s_rank[1]);
            lo = s_rank[2];
            hi = s_rank[3];
        }
        summary[SMOE_DIAG_ACTIVE_EXPERTS] = a;
        summary[SMOE_DIAG_NORM_MEDIAN] = med;
        summary[SMOE_DIAG_NORM_MAX_TO_MEDIAN] = med > 0.f ? hi / med : 0.f;
        summary[SMOE_DIAG_NORM_MIN_TO_MEDIAN] = med > 0.f ? lo / med : 0.f;
        summary[SMOE_DIAG_CONF_MEAN] = cs / (float)T;
        summary[SMOE_DIAG_CONF_MIN] = cn;
        summary[SMOE_DIAG_LOAD_MAX_TO_MEAN] = cm / ((float)routed / (float)E);
        summary[SMOE_DIAG_NORM_PEAK] = nm;
    }
}

}  // namespace

cudaError_t launch_diag(const smoe_config_t& c, int64_t T, const float* row_norm, const int32_t* offsets,
                        const float* conf, int32_t* count, float* norm_mean, float* norm_max, float* summary,
                        int32_t* err, cudaStream_t s) {
    cudaError_t e;
    {
        LaunchTimer lt(K_DIAG, s);
        e = launch_pdl(diag_kernel, dim3(1), dim3(kDiagThreads), 0, s, row_norm, offsets, conf, c.n_experts, (int)T,
                       c.top_k, count, norm_mean, norm_max, summary, err);
    }
    if (e == cudaSuccess) launches_add(1);
    return e;
}

}  // namespace smoe
