// Expert FFNs on the 5th-generation tensor cores: a persistent, warp-specialised grouped GEMM
// (TMA -> shared memory -> tcgen05.mma -> TMEM -> epilogue) used twice per layer:
//   gate/up:  h = SiLU(X W_g^T) * (X W_u^T)   (both projections in one pass, fused epilogue)
//   down:     y = h W_d^T
// Source: SwiGLU experts with gate and up projections (Step 3.5 Flash summary, paperlayer.ai,
// §B "Detail Analysis of Localized Activation Blow-up"); widths from the model card's raw
// config fields moe_intermediate_size 1280 and share_expert_dim 1280; 288 routed experts +
// 1 shared expert per token (hyper.ai summary, section "方法").
//
// Operand orientation ("swap AB"): the MMA's M side is 128 weight rows (output features) and
// its N side is a tile of NT token rows of one expert group, so a decode step with ~2 tokens
// per expert still runs full 128-row MMAs (N = 16), and the weight tile of an expert streams
// from HBM once per token tile. D[feature, token] lives in TMEM, lane = feature.
//
// Groups 0..E-1: routed experts, rows offsets[g] .. offsets[g+1] of the permuted activations.
// Group E: the shared expert over all T rows (x for gate/up, the last T rows of h for down).
// Work unit = (group, 128-feature block mb, token tile nb), enumerated group-major, then mb,
// then nb; CTA i takes units i, i + grid, ... (static persistent schedule, grid = #SMs).
//
// Roles (192 threads): warp 0 lane 0 issues TMA loads into an S-stage ring; warp 1 lane 0
// issues tcgen05.mma (M=128, N=NT, K=16 per instruction, 4 per 64-wide stage; for gate/up a
// second MMA into the neighbouring TMEM columns) and commits stage and accumulator barriers;
// warps 2-5 drain the accumulator (tcgen05.ld, warp w reads TMEM lanes 32*(w%4)..+31),
// apply SiLU(g)*u or pass through, round to bf16 and store. Accumulators are double-buffered
// in TMEM whenever two fit in 512 columns, so the epilogue overlaps the next unit's MMAs.
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace smoe {

namespace {

constexpr int kBK = 64;             // K elements per stage: 128 bytes of bf16 = one swizzle row
constexpr int kThreads = 192;
constexpr int kTmemCols = 512;
constexpr int kSmemBudget = 200 * 1024;

template <int NT, bool DUAL>
struct GemmCfg {
    static constexpr int A_ROWS = DUAL ? 256 : 128;     // gate 128 + up 128, or 128
    static constexpr int A_BYTES = A_ROWS * 128;
    static constexpr int B_BYTES = NT * 128;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGES = (kSmemBudget / STAGE_BYTES) > 12 ? 12 : (kSmemBudget / STAGE_BYTES);
    static constexpr int ACC_COLS = DUAL ? 2 * NT : NT;
    static constexpr int NACC = (2 * ACC_COLS <= kTmemCols) ? 2 : 1;
    static_assert(NT % 16 == 0 && NT >= 16 && NT <= 256, "MMA N for M=128 is 16..256 in steps of 16");
    static_assert(ACC_COLS <= kTmemCols, "accumulator must fit TMEM");
    static_assert(STAGES >= 2, "need at least two stages");
};

struct GemmParams {
    const int32_t* offsets;   // [E+1] routed row offsets
    int E;                    // routed experts (group E = shared expert)
    int T;                    // tokens (rows of the shared group)
    int routed_rows;          // T*k: rows of the routed activations
    int K;                    // reduction length
    int n_out;                // output features per group (= leading dimension of out)
    int shared_in_row;        // first activation row of the shared group in its tensor map
    int shared_out_row;       // first output row of the shared group (= T*k)
    uint16_t* out;            // [*, n_out] bf16
    int32_t* err;
};

template <int NT, bool DUAL>
size_t gemm_smem_bytes(int E) {
    using C = GemmCfg<NT, DUAL>;
    size_t b = 1024;                                   // alignment slack
    b += (size_t)C::STAGES * C::STAGE_BYTES;
    b += sizeof(uint64_t) * (2 * C::STAGES + 5);       // full, empty, tfull[2], tempty[2], drain
    b += 16;                                           // tmem slot, abort flag
    b += sizeof(int32_t) * (2 * (size_t)E + 3);        // prefix[E+2], offs[E+1]
    return b;
}

struct Unit {
    int g, mb, nb;
};

__device__ __forceinline__ int group_rows(int g, int E, int T, const int32_t* offs) {
    return g < E ? offs[g + 1] - offs[g] : T;
}

__device__ __forceinline__ Unit decode_unit(int u, const int32_t* prefix, const int32_t* offs, int E, int T, int NT) {
    int lo = 0, hi = E;   // find g with prefix[g] <= u < prefix[g+1]
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= u) lo = mid; else hi = mid - 1;
    }
    const int g = lo;
    const int nblk = (group_rows(g, E, T, offs) + NT - 1) / NT;
    const int local = u - prefix[g];
    return Unit{g, local / nblk, local % nblk};
}

template <int NT, bool DUAL>
__global__ void __launch_bounds__(kThreads, 1)
expert_gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_act,
                   const __grid_constant__ CUtensorMap tm_sh, const GemmParams p) {
    using C = GemmCfg<NT, DUAL>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(tiles + (size_t)C::STAGES * C::STAGE_BYTES);
    uint64_t* empty = full + C::STAGES;
    uint64_t* tfull = empty + C::STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int32_t* prefix = reinterpret_cast<int32_t*>(tmem_slot + 4);   // [E+2]
    int32_t* offs = prefix + (p.E + 2);                              // [E+1]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = p.E;
    const int MB = p.n_out / 128;
    const int KB = p.K / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tfull[a]), 1);
            mbar_init(smem_u32(&tempty[a]), 128);
        }
        mbar_init(smem_u32(drain), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    if (warp == 1 && lane == 0) {
        tma_prefetch_desc(&tm_w);
        tma_prefetch_desc(&tm_act);
        tma_prefetch_desc(&tm_sh);
    }
    if (warp == 2) {
        // group table: offsets (validated), then units per group and their exclusive prefix
        bool bad = false;
        for (int i = lane; i <= E; i += 32) {
            int v = p.offsets[i];
            if (v < 0 || v > p.routed_rows) { bad = true; v = 0; }
            offs[i] = v;
        }
        __syncwarp();
        for (int i = lane; i < E; i += 32)
            if (offs[i + 1] < offs[i]) bad = true;
        if (__any_sync(0xFFFFFFFFu, bad)) {
            // corrupt offsets: run no routed work (shared expert only)
            for (int i = lane; i <= E; i += 32) offs[i] = 0;
            if (lane == 0) record_error(p.err, SMOE_ERR_DEVICE);
        }
        __syncwarp();
        const int ngroups = E + 1;
        const int chunk = (ngroups + 31) / 32;
        const int g0 = min(lane * chunk, ngroups), g1 = min(g0 + chunk, ngroups);
        int local = 0;
        for (int g = g0; g < g1; ++g) local += ((group_rows(g, E, p.T, offs) + NT - 1) / NT) * MB;
        int incl = local;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int n = __shfl_up_sync(0xFFFFFFFFu, incl, off);
            if (lane >= off) incl += n;
        }
        int run = incl - local;
        for (int g = g0; g < g1; ++g) {
            prefix[g] = run;
            run += ((group_rows(g, E, p.T, offs) + NT - 1) / NT) * MB;
        }
        if (lane == 31) prefix[E + 1] = incl;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total = prefix[E + 1];

    if (warp == 0 && lane == 0) {
        // ---------------------------------------------------------------- TMA producer
        const uint64_t pol_w = l2_policy_evict_first();
        const uint64_t pol_a = l2_policy_evict_last();
        int stage = 0;
        uint32_t phase = 0, armed = 0, armed_par = 0;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < total; u += gridDim.x) {
            const Unit w = decode_unit(u, prefix, offs, E, p.T, NT);
            const int a_row = DUAL ? (w.g * MB + w.mb) * 256 : w.g * p.n_out + w.mb * 128;
            const int b_row = (w.g < E ? offs[w.g] : p.shared_in_row) + w.nb * NT;
            const CUtensorMap* bm = (w.g < E) ? &tm_act : &tm_sh;
            for (int kb = 0; kb < KB; ++kb) {
                if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, p.err, abort_flag, true)) { ok = false; break; }
                const uint32_t fb = smem_u32(&full[stage]);
                mbar_arrive_expect_tx(fb, C::STAGE_BYTES);
                uint8_t* a_s = tiles + (size_t)stage * C::STAGE_BYTES;
                tma_load_2d(smem_u32(a_s), &tm_w, kb * kBK, a_row, fb, pol_w);
                tma_load_2d(smem_u32(a_s + C::A_BYTES), bm, kb * kBK, b_row, fb, pol_a);
                armed |= 1u << stage;
                armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
            }
        }
        // every load issued must land before the CTA may exit
        for (int s = 0; s < C::STAGES; ++s)
            if ((armed >> s) & 1u) mbar_wait(smem_u32(&full[s]), (armed_par >> s) & 1u, p.err, abort_flag, false);
    } else if (warp == 1 && lane == 0) {
        // ---------------------------------------------------------------- MMA issuer
        constexpr uint32_t idesc = idesc_bf16_f32(128, NT);
        int stage = 0, acc = 0;
        uint32_t phase = 0, acc_phase = 0;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < total; u += gridDim.x) {
            if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1u, p.err, abort_flag, true)) break;
            tc_fence_after();
            const uint32_t d = tmem_base + (uint32_t)(acc * C::ACC_COLS);
            for (int kb = 0; kb < KB; ++kb) {
                if (!mbar_wait(smem_u32(&full[stage]), phase, p.err, abort_flag, true)) { ok = false; break; }
                tc_fence_after();
                const uint32_t a_s = smem_u32(tiles + (size_t)stage * C::STAGE_BYTES);
                const uint32_t b_s = a_s + C::A_BYTES;
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk) {
                    const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
                    const uint64_t bdesc = smem_desc_sw128(b_s + kk * 32);
                    umma_f16_ss(d, smem_desc_sw128(a_s + kk * 32), bdesc, idesc, accum);
                    if (DUAL) umma_f16_ss(d + NT, smem_desc_sw128(a_s + 16384 + kk * 32), bdesc, idesc, accum);
                }
                umma_commit(smem_u32(&empty[stage]));
                if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
            umma_commit(smem_u32(&tfull[acc]));
            if (C::NACC == 2) {
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            } else {
                acc_phase ^= 1u;
            }
        }
        // all MMAs issued by this thread must finish before TMEM is released
        umma_commit(smem_u32(drain));
        mbar_wait(smem_u32(drain), 0u, p.err, abort_flag, false);
    } else if (warp >= 2) {
        // ---------------------------------------------------------------- epilogue
        const int q = warp & 3;            // TMEM lane quadrant this warp may access
        const int row = q * 32 + lane;     // accumulator row = output feature within the block
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int u = blockIdx.x; u < total; u += gridDim.x) {
            const Unit w = decode_unit(u, prefix, offs, E, p.T, NT);
            const int rows = group_rows(w.g, E, p.T, offs);
            const int out_base = (w.g < E ? offs[w.g] : p.shared_out_row) + w.nb * NT;
            const int nvalid = min(NT, rows - w.nb * NT);
            if (!mbar_wait(smem_u32(&tfull[acc]), acc_phase, p.err, abort_flag, true)) break;
            tc_fence_after();
            const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * C::ACC_COLS);
            uint16_t* dst = p.out + (size_t)out_base * p.n_out + w.mb * 128 + row;
            for (int c0 = 0; c0 < nvalid; c0 += 16) {
                uint32_t g16[16], u16[16];
                if (DUAL)
                    tmem_ld2_x16_wait(t_row + c0, t_row + NT + c0, g16, u16);
                else
                    tmem_ld_x16_wait(t_row + c0, g16);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    if (c0 + j < nvalid) {
                        const float gv = __uint_as_float(g16[j]);
                        float v = gv;
                        if (DUAL) v = (gv / (1.0f + expf(-gv))) * __uint_as_float(u16[j]);
                        dst[(size_t)(c0 + j) * p.n_out] = float_to_bf16_bits(v);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&tempty[acc]));
            if (C::NACC == 2) {
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            } else {
                acc_phase ^= 1u;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// ------------------------------------------------------------------------------------------
// host side: tensor maps through the driver entry point (no link-time libcuda dependency)
// ------------------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2D bf16 tensor [rows][cols] row-major; box = 64 columns (128 bytes) x box_rows, 128B swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NT, bool DUAL>
cudaError_t run_gemm(const CUtensorMap& w, const CUtensorMap& act, const CUtensorMap& sh, const GemmParams& p,
                     int grid, cudaStream_t s) {
    const size_t smem = gemm_smem_bytes<NT, DUAL>(p.E);
    cudaError_t e = cudaFuncSetAttribute(expert_gemm_kernel<NT, DUAL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    {
        LaunchTimer lt(DUAL ? K_EXPERT_GATEUP : K_EXPERT_DOWN, s);
        expert_gemm_kernel<NT, DUAL><<<grid, kThreads, smem, s>>>(w, act, sh, p);
    }
    return cudaGetLastError();
}

template <bool DUAL>
cudaError_t dispatch_nt(int nt, const CUtensorMap& w, const CUtensorMap& act, const CUtensorMap& sh,
                        const GemmParams& p, int grid, cudaStream_t s) {
    switch (nt) {
        case 16: return run_gemm<16, DUAL>(w, act, sh, p, grid, s);
        case 32: return run_gemm<32, DUAL>(w, act, sh, p, grid, s);
        case 64: return run_gemm<64, DUAL>(w, act, sh, p, grid, s);
        case 128: return run_gemm<128, DUAL>(w, act, sh, p, grid, s);
        default: return run_gemm<256, DUAL>(w, act, sh, p, grid, s);
    }
}

}  // namespace

// Token tile: the smallest power of two >= 1.25 x the mean rows per routed expert, 16..256.
int choose_token_tile(const smoe_config_t& c, int64_t T) {
    const double mean = (double)T * c.top_k / c.n_experts;
    int nt = 16;
    while (nt < 256 && nt < 1.25 * mean) nt *= 2;
    return nt;
}

size_t packed_gateup_bytes(const smoe_config_t& c) {
    return (size_t)(c.n_experts + 1) * 2 * c.inter * c.hidden * 2;
}
size_t packed_down_bytes(const smoe_config_t& c) { return (size_t)(c.n_experts + 1) * c.hidden * c.inter * 2; }

cudaError_t launch_expert_ffn(const smoe_config_t& c, const uint16_t* x, const uint16_t* x_perm,
                              const int32_t* offsets, int64_t T, const void* packed, uint16_t* y, uint16_t* h,
                              int32_t* err, int num_sms, cudaStream_t s) {
    const int E = c.n_experts, H = c.hidden, I = c.inter, k = c.top_k;
    const int64_t routed = T * k;
    const int nt = choose_token_tile(c, T);
    const uint8_t* wgu = static_cast<const uint8_t*>(packed);
    const uint8_t* wdn = wgu + packed_gateup_bytes(c);

    CUtensorMap m_wgu, m_xp, m_x, m_wd, m_h;
    if (!make_map(&m_wgu, wgu, (uint64_t)(E + 1) * 2 * I, H, 256) ||
        !make_map(&m_xp, x_perm, (uint64_t)routed, H, nt) || !make_map(&m_x, x, (uint64_t)T, H, nt) ||
        !make_map(&m_wd, wdn, (uint64_t)(E + 1) * H, I, 128) ||
        !make_map(&m_h, h, (uint64_t)(routed + T), I, nt))
        return cudaErrorNotSupported;

    GemmParams p1{offsets, E, (int)T, (int)routed, H, I, 0, (int)routed, h, err};
    cudaError_t e = dispatch_nt<true>(nt, m_wgu, m_xp, m_x, p1, num_sms, s);
    if (e != cudaSuccess) return e;
    GemmParams p2{offsets, E, (int)T, (int)routed, I, H, (int)routed, (int)routed, y, err};
    e = dispatch_nt<false>(nt, m_wd, m_h, m_h, p2, num_sms, s);
    if (e == cudaSuccess) launches_add(2);
    return e;
}

}  // namespace smoe
