// Token -> expert dispatch: per-block expert histograms, a column scan, and a stable scatter
// that orders rows by expert, then token, then slot (a unique order, so the result is
// bit-exact and independent of scheduling), plus an optional gather of x into x_perm.
//
// Source: sparse top-k routing, Step 3.5 Flash summary (hyper.ai), section "方法" (method):
// each token is sent to 8 of 288 routed experts; the grouping by expert is what the grouped
// expert GEMMs consume.
//
// Kernels:
//   permute_hist_kernel    block b counts entries of tokens [256 b, 256 b + 256) per expert
//   permute_scan_kernel    one CTA: per-expert exclusive scan over blocks, counts, offsets
//   permute_scatter_kernel rank of (t, e) among the block's tokens that chose e: per-warp
//                          lane bitmasks in shared memory (a token picks an expert at most
//                          once), warp prefix over the block, block base from the scan
//   gather_rows_kernel     x_perm[r] = x[row_token[r]], one warp per row, 16-byte accesses
//   permute_small_kernel   T <= 1024: histogram, scan and scatter in one CTA (same results)
// An expert id outside [0, E) or repeated within a token is skipped (perm_row = -1) and
// recorded as SMOE_ERR_DEVICE.
#include "common.cuh"
#include "internal.h"

namespace smoe {

namespace {

constexpr int TB = kPermuteTokensPerBlock;   // tokens per block = threads per block
constexpr int WARPS = TB / 32;

// Entry (t, j) is valid when its expert is in range and not already chosen at an earlier slot.
__device__ __forceinline__ bool entry_valid(const int32_t* idx, int t, int j, int k, int E, int32_t* err) {
    const int e = idx[(size_t)t * k + j];
    if (e < 0 || e >= E) {
        record_error(err, SMOE_ERR_DEVICE);
        return false;
    }
    for (int q = 0; q < j; ++q) {
        if (idx[(size_t)t * k + q] == e) {
            record_error(err, SMOE_ERR_DEVICE);
            return false;
        }
    }
    return true;
}

__global__ void __launch_bounds__(TB) permute_hist_kernel(const int32_t* __restrict__ idx, int T, int k, int E,
                                                          int32_t* __restrict__ hist, int32_t* err) {
    pdl_wait();
    pdl_launch_dependents();
    extern __shared__ int32_t sh[];
    for (int e = threadIdx.x; e < E; e += TB) sh[e] = 0;
    __syncthreads();
    const int t = blockIdx.x * TB + threadIdx.x;
    if (t < T) {
        for (int j = 0; j < k; ++j)
            if (entry_valid(idx, t, j, k, E, err)) atomicAdd(&sh[idx[(size_t)t * k + j]], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += TB) hist[(size_t)blockIdx.x * E + e] = sh[e];
}

// One CTA of 1024 threads: base[b][e] = sum_{b' < b} hist[b'][e]; counts[e]; offsets = scan.
__global__ void __launch_bounds__(1024) permute_scan_kernel(const int32_t* __restrict__ hist, int nblk, int E,
                                                            int32_t* __restrict__ base, int32_t* __restrict__ counts,
                                                            int32_t* __restrict__ offsets) {
    pdl_wait();
    pdl_launch_dependents();
    __shared__ int32_t warp_tot[32];
    const int e = threadIdx.x;
    int32_t run = 0;
    if (e < E) {
        for (int b = 0; b < nblk; ++b) {
            base[(size_t)b * E + e] = run;
            run += hist[(size_t)b * E + e];
        }
        counts[e] = run;
    }
    // exclusive scan of run over e (E <= 1024)
    const int lane = e & 31, w = e >> 5;
    int32_t v = run;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int32_t n = __shfl_up_sync(0xFFFFFFFFu, v, off);
        if (lane >= off) v += n;
    }
    if (lane == 31) warp_tot[w] = v;
    __syncthreads();
    if (w == 0) {
        int32_t tv = warp_tot[lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int32_t n = __shfl_up_sync(0xFFFFFFFFu, tv, off);
            if (lane >= off) tv += n;
        }
        warp_tot[lane] = tv;   // inclusive totals of warps 0..lane
    }
    __syncthreads();
    const int32_t incl = v + (w > 0 ? warp_tot[w - 1] : 0);
    if (e < E) offsets[e] = incl - run;
    if (e == E - 1) offsets[E] = incl;
}

__global__ void __launch_bounds__(TB) permute_scatter_kernel(const int32_t* __restrict__ idx, int T, int k, int E,
                                                             const int32_t* __restrict__ base,
                                                             const int32_t* __restrict__ offsets,
                                                             int32_t* __restrict__ perm_row,
                                                             int32_t* __restrict__ row_token, int32_t* err) {
    pdl_wait();
    pdl_launch_dependents();
    extern __shared__ uint32_t smem[];
    uint32_t* wmask = smem;                                        // [WARPS][E]
    int32_t* wbase = reinterpret_cast<int32_t*>(smem + WARPS * E);  // [WARPS][E]
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < WARPS * E; i += TB) wmask[i] = 0u;
    __syncthreads();
    const int t = blockIdx.x * TB + threadIdx.x;
    if (t < T) {
        for (int j = 0; j < k; ++j) {
            // duplicates/out-of-range are recorded by the histogram pass; skip them silently here
            const int e = idx[(size_t)t * k + j];
            bool ok = (e >= 0 && e < E);
            for (int q = 0; ok && q < j; ++q) ok = idx[(size_t)t * k + q] != e;
            if (ok) atomicOr(&wmask[w * E + e], 1u << lane);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += TB) {
        int32_t run = offsets[e] + base[(size_t)blockIdx.x * E + e];
        for (int q = 0; q < WARPS; ++q) {
            wbase[q * E + e] = run;
            run += __popc(wmask[q * E + e]);
        }
    }
    __syncthreads();
    if (t < T) {
        const uint32_t below = (1u << lane) - 1u;
        for (int j = 0; j < k; ++j) {
            const int e = idx[(size_t)t * k + j];
            bool ok = (e >= 0 && e < E);
            for (int q = 0; ok && q < j; ++q) ok = idx[(size_t)t * k + q] != e;
            int32_t row = -1;
            if (ok) {
                row = wbase[w * E + e] + __popc(wmask[w * E + e] & below);
                row_token[row] = t;
            }
            perm_row[(size_t)t * k + j] = row;
        }
    }
    (void)err;
}

// The whole permutation in one CTA of up to 1024 threads (one token per thread), for T <= 1024:
// the same histogram, scan and stable rank as the three kernels above, kept in shared memory.
// Outputs are identical to the multi-block path.
constexpr int kSmallThreads = 1024;
constexpr int kSmallWarps = kSmallThreads / 32;

__global__ void __launch_bounds__(kSmallThreads) permute_small_kernel(const int32_t* __restrict__ idx, int T, int k,
                                                                      int E, int32_t* __restrict__ counts,
                                                                      int32_t* __restrict__ offsets,
                                                                      int32_t* __restrict__ perm_row,
                                                                      int32_t* __restrict__ row_token, int32_t* err,
                                                                      int early_trigger) {
    // early_trigger: the next kernel may launch at once (its own wait still covers this one)
    if (early_trigger) pdl_launch_dependents();
    pdl_wait();
    if (!early_trigger) pdl_launch_dependents();
    extern __shared__ uint32_t smem[];
    uint32_t* wmask = smem;                                                  // [warps][E]
    int32_t* wbase = reinterpret_cast<int32_t*>(smem + kSmallWarps * E);     // [warps][E]
    int32_t* offs = wbase + kSmallWarps * E;                                 // [E + 1]
    __shared__ int32_t warp_tot[32];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < kSmallWarps * E; i += kSmallThreads) wmask[i] = 0u;
    __syncthreads();
    const int t = threadIdx.x;
    if (t < T) {
        for (int j = 0; j < k; ++j)
            if (entry_valid(idx, t, j, k, E, err)) atomicOr(&wmask[w * E + idx[(size_t)t * k + j]], 1u << lane);
    }
    __syncthreads();
    // per-expert warp prefix and totals; then an exclusive scan over experts (E <= 1024)
    int32_t cnt = 0;
    const int e = threadIdx.x;
    if (e < E) {
        for (int q = 0; q < kSmallWarps; ++q) {
            wbase[q * E + e] = cnt;
            cnt += __popc(wmask[q * E + e]);
        }
        counts[e] = cnt;
    }
    int32_t v = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int32_t n = __shfl_up_sync(0xFFFFFFFFu, v, off);
        if (lane >= off) v += n;
    }
    if (lane == 31) warp_tot[w] = v;
    __syncthreads();
    if (w == 0) {
        int32_t tv = warp_tot[lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int32_t n = __shfl_up_sync(0xFFFFFFFFu, tv, off);
            if (lane >= off) tv += n;
        }
        warp_tot[lane] = tv;
    }
    __syncthreads();
    const int32_t incl = v + (w > 0 ? warp_tot[w - 1] : 0);
    if (e < E) {
        offs[e] = incl - cnt;
        offsets[e] = incl - cnt;
    }
    if (e == E - 1) offsets[E] = incl;
    __syncthreads();
    if (t < T) {
        const uint32_t below = (1u << lane) - 1u;
        for (int j = 0; j < k; ++j) {
            const int ex = idx[(size_t)t * k + j];
            bool ok = (ex >= 0 && ex < E);
            for (int q = 0; ok && q < j; ++q) ok = idx[(size_t)t * k + q] != ex;
            int32_t row = -1;
            if (ok) {
                row = offs[ex] + wbase[w * E + ex] + __popc(wmask[w * E + ex] & below);
                row_token[row] = t;
            }
            perm_row[(size_t)t * k + j] = row;
        }
    }
}

size_t permute_small_smem(int E) { return (2 * (size_t)kSmallWarps * E + E + 1) * sizeof(int32_t); }

// x_perm[r] = x[row_token[r]] for r < offsets[E]; one warp per row.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint16_t* __restrict__ x,
                                                          const int32_t* __restrict__ row_token,
                                                          const int32_t* __restrict__ offsets, int E, int T, int H,
                                                          uint16_t* __restrict__ x_perm, int32_t* err) {
    pdl_wait();
    pdl_launch_dependents();
    const int nrows = offsets[E];
    const int lane = threadIdx.x & 31;
    const int vec = H / 8;
    // each row of x is read k times and x fits in L2, while the T*k copies stream out once: keep
    // x in L2 (evict-last) and let the copies pass through (evict-first), so the write stream
    // does not push x out and make every copy re-read it from HBM
    const uint64_t keep = l2_policy_evict_last(), pass = l2_policy_evict_first();
    for (int r = blockIdx.x * 8 + (threadIdx.x >> 5); r < nrows; r += gridDim.x * 8) {
        const int t = row_token[r];
        if (t < 0 || t >= T) {
            if (lane == 0) record_error(err, SMOE_ERR_DEVICE);
            continue;
        }
        const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H);
        uint4* dst = reinterpret_cast<uint4*>(x_perm + (size_t)r * H);
        int c = lane;
        for (; c + 224 < vec; c += 256) {   // eight 16-byte vectors in flight per lane
            uint4 v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = ld_global_hint(src + c + 32 * i, keep);
#pragma unroll
            for (int i = 0; i < 8; ++i) st_global_hint(dst + c + 32 * i, v[i], pass);
        }
        for (; c < vec; c += 32) st_global_hint(dst + c, ld_global_hint(src + c, keep), pass);
    }
}

}  // namespace

cudaError_t launch_permute(const smoe_config_t& c, const int32_t* topk_idx, int64_t T, const uint16_t* x,
                           int32_t* counts, int32_t* offsets, int32_t* perm_row, int32_t* row_token,
                           uint16_t* x_perm, int32_t* hist, int32_t* base, int32_t* err, cudaStream_t s,
                           int gather_cols, bool early_trigger) {
    const int E = c.n_experts, k = c.top_k;
    const int nblk = (int)((T + TB - 1) / TB);
    cudaError_t e;
    int n = 3;
    const size_t small_sm = permute_small_smem(E);
    if (T <= kSmallThreads && small_sm <= 200 * 1024) {
        if (small_sm > 48 * 1024) {
            e = cudaFuncSetAttribute(permute_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)small_sm);
            if (e != cudaSuccess) return e;
        }
        {
            LaunchTimer lt(K_PERMUTE_SCATTER, s);
            e = launch_pdl(permute_small_kernel, dim3(1), dim3(kSmallThreads), small_sm, s, topk_idx, (int)T, k, E,
                           counts, offsets, perm_row, row_token, err, early_trigger ? 1 : 0);
        }
        if (e != cudaSuccess) return e;
        n = 1;
    } else {
        {
            LaunchTimer lt(K_PERMUTE_HIST, s);
            e = launch_pdl(permute_hist_kernel, dim3(nblk), dim3(TB), E * sizeof(int32_t), s, topk_idx, (int)T, k, E,
                           hist, err);
        }
        if (e != cudaSuccess) return e;
        {
            LaunchTimer lt(K_PERMUTE_SCAN, s);
            e = launch_pdl(permute_scan_kernel, dim3(1), dim3(1024), 0, s, (const int32_t*)hist, nblk, E, base, counts,
                           offsets);
        }
        if (e != cudaSuccess) return e;
        const size_t sm = 2 * WARPS * E * sizeof(uint32_t);
        if (sm > 48 * 1024) {
            e = cudaFuncSetAttribute(permute_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
            if (e != cudaSuccess) return e;
        }
        {
            LaunchTimer lt(K_PERMUTE_SCATTER, s);
            e = launch_pdl(permute_scatter_kernel, dim3(nblk), dim3(TB), sm, s, topk_idx, (int)T, k, E,
                           (const int32_t*)base, (const int32_t*)offsets, perm_row, row_token, err);
        }
        if (e != cudaSuccess) return e;
    }
    if (x != nullptr && x_perm != nullptr) {
        const int64_t rows = T * k;
        int64_t blocks = (rows + 7) / 8;
        if (blocks > 148 * 32) blocks = 148 * 32;
        {
            LaunchTimer lt(K_GATHER_ROWS, s);
            e = launch_pdl(gather_rows_kernel, dim3((unsigned)blocks), dim3(256), 0, s, x, (const int32_t*)row_token,
                           (const int32_t*)offsets, E, (int)T, gather_cols > 0 ? gather_cols : c.hidden, x_perm, err);
        }
        if (e != cudaSuccess) return e;
        ++n;
    }
    launches_add(n);
    return cudaSuccess;
}

}  // namespace smoe
