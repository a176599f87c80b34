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
// Token tile per group: the smallest power of two >= the group's row count, between 16 and a
// launch-wide maximum NT_MAX (so an expert with 2 tokens runs N=16 MMAs while a hot expert with
// 1000 tokens runs N=256 tiles). One TMA tensor map per tile height loads exactly that box.
// Work unit = (token tile (group, nb), 128-feature block mb). The token tiles are listed in
// group order and the units dealt to the CTAs in snake order (static persistent schedule,
// grid = #SMs): see the work table below.
//
// Roles (192 threads): warp 0 lane 0 issues TMA loads into an S-stage ring of BK-wide K slices
// (BK = 64: 128-byte swizzled rows; the ring fills the 227 KB of shared memory);
// warp 1 lane 0 issues tcgen05.mma (M=128, N=tile, K=16 per instruction; for gate/up a second
// MMA into the neighbouring TMEM columns) and commits stage and accumulator barriers; warps 2-5
// drain the accumulator (tcgen05.ld, warp w reads TMEM lanes 32*(w%4)..+31), apply SiLU(g)*u or
// pass through, round to bf16 and store. Accumulators are double-buffered in TMEM whenever two
// fit in 512 columns, so the epilogue overlaps the next unit's MMAs.
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace smoe {

namespace {

// K elements per pipeline stage of the bf16 kernels: 64 = one 128-byte swizzled row, the width
// of a packed weight tile (stages of 32 and 16 measured slower and are not built).
#define SMOE_GEMM_BK 64
#ifndef SMOE_MAX_TOKEN_TILE
#define SMOE_MAX_TOKEN_TILE 256  // cap on the token tile (a tuning constant)
#endif
// 256 is also the largest MMA N, the largest box height of a TMA map (kNumTiles maps, 16..256),
// and the most rows the producer warp's lanes cover with one four-row gather each per CTA half
static_assert(SMOE_MAX_TOKEN_TILE >= 16 && SMOE_MAX_TOKEN_TILE <= 256, "token tile cap in 16..256");

constexpr int kThreads = 192;
constexpr int kTmemCols = 512;
constexpr int kNumTiles = 5;     // token tiles 16, 32, 64, 128, 256
#ifndef SMOE_MAX_STAGES
#define SMOE_MAX_STAGES 24       // cap on the pipeline depth (a tuning constant, <= 32)
#endif
constexpr int kMaxStages = SMOE_MAX_STAGES;
#ifndef SMOE_PAIR_MIN_TILE
#define SMOE_PAIR_MIN_TILE 64    // CTA pairs for launches whose largest token tile is at least this
#endif
constexpr int kPairMinTile = SMOE_PAIR_MIN_TILE;
#ifndef SMOE_PAIR_EPI_WARPS
#define SMOE_PAIR_EPI_WARPS 8    // epilogue warps of a CTA-pair gate/up CTA: 4, 8 or 16
#endif
#ifndef SMOE_PAIR_EPI_WARPS_DOWN
#define SMOE_PAIR_EPI_WARPS_DOWN 8   // the same for the down GEMM
#endif

struct GemmMaps {
    CUtensorMap w;                  // weights [rows][K]: box {BK, 256 (gate/up) or 128 (down)}
    CUtensorMap act[kNumTiles];     // routed activations [T*k][K]: box {BK, 16 << i}
    CUtensorMap sh[kNumTiles];      // shared-group activations: box {BK, 16 << i}
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
    int nt_max;               // largest token tile of this launch (16..256, power of two)
    int stages;               // pipeline depth
    int k_wrap;               // B's K coordinate wraps every k_wrap blocks (0 = no wrap)
    int out_ld;               // leading dimension of the output rows
    int out_valid;            // output features stored: f < out_valid
    const int32_t* row_token; // gather mode (routed groups read x rows by token), else nullptr
    float clamp_routed;       // SwiGLU clamp limit of routed groups (0 = off)
    float clamp_shared;       // SwiGLU clamp limit of the shared group (0 = off)
    int ksplit;               // K split into this many equal ranges, one unit each (router pieces)
    size_t split_stride;      // elements between the partial outputs of consecutive K ranges
    uint16_t* out;            // [*, out_ld] bf16 (gate/up, down)
    float* out_f32;           // [*, out_ld] fp32 (router)
    int32_t* err;
    int max_tiles;            // capacity of the token-tile table in shared memory
    // e4m3 launches: acc * w_scale[feature] * act_scale[activation row's token or row]
    const float* w_scale;     // gate/up: [E+1][2][n_out] (gate rows, then up rows); down: [E+1][n_out]
    const float* act_scale;   // per token (gate/up) or per activation row (down)
    const int32_t* scale_tok; // gate/up: routed activation row -> token (act_scale index); down: nullptr
    int scale_shared_base;    // act_scale index of the shared group's first row (0, or T*k for down)
    int shared_first = 0;     // list the shared group's tiles before the routed groups' (else after)
    int shared_prewait = 0;   // single-CTA kernel: the shared group's units run before the dependency
                              // wait (its inputs must not come from the kernels just before this one)
};

// What a launch computes: the down projection, the fused gate/up + SiLU*mul, or router logits.
enum GemmMode { MODE_DOWN = 0, MODE_GATEUP = 1, MODE_ROUTER = 2 };

// CTA-pair kernels: producer warp, MMA warp and the epilogue warps of their mode
template <int MODE>
__host__ __device__ constexpr int pair_epi_warps() { return MODE == MODE_DOWN ? SMOE_PAIR_EPI_WARPS_DOWN : SMOE_PAIR_EPI_WARPS; }
template <int MODE>
__host__ __device__ constexpr int pair_threads() { return 64 + 32 * pair_epi_warps<MODE>(); }

template <int MODE, int BK>
struct GemmCfg {
    static constexpr bool DUAL = MODE == MODE_GATEUP;
    static constexpr int SW = BK * 2;                     // bytes per swizzled row
    static constexpr int A_ROWS = DUAL ? 256 : 128;       // gate 128 + up 128, or 128
    static constexpr int A_BYTES = A_ROWS * SW;
    static constexpr int UP_OFFSET = 128 * SW;            // up rows inside the A tile
    static_assert(BK == 64, "stage K width: one 128-byte row of a packed tile");
};

__host__ __device__ inline int stage_bytes(bool dual, int bk, int nt_max) {
    return (dual ? 256 : 128) * bk * 2 + nt_max * bk * 2;
}

// Upper bound on the token tiles of a launch: a group of r rows has one tile if r <= nt_max,
// else ceil(r / nt_max) <= r / nt_max + 1, and the rows of all groups add up to at most
// routed_rows + T.
__host__ __device__ inline int max_token_tiles(int E, int routed_rows, int T, int nt_max) {
    return E + 2 + (routed_rows + T) / nt_max;
}

__host__ __device__ inline size_t gemm_smem_bytes(int stages, int stage_b, int E, int max_tiles) {
    size_t b = 1024;                                       // alignment slack
    b += (size_t)stages * stage_b;
    b += sizeof(uint64_t) * (2 * (size_t)stages + 6);      // full, empty, tfull[2], tempty[2], drain, tab_ready
    b += 16;                                               // tmem slot, abort flag, tile count
    b += sizeof(int32_t) * ((size_t)max_tiles + E + 1);    // tiles[max_tiles], offs[E+1]
    return b;
}

struct Unit {
    int g, mb, nb, nt;
};

__device__ __forceinline__ int group_rows(int g, int E, int T, const int32_t* offs) {
    return g < E ? offs[g + 1] - offs[g] : T;
}

// Token tile of a group: smallest power of two >= rows, clamped to [16, nt_max].
__device__ __forceinline__ int group_tile(int rows, int nt_max) {
    int nt = 16;
    while (nt < rows && nt < nt_max) nt <<= 1;
    return nt;
}

__device__ __forceinline__ int tile_index(int nt) { return 31 - __clz(nt) - 4; }   // 16 -> 0 ... 256 -> 4

// Columns the MMAs of a unit compute: its valid token rows rounded up to 16 (the N step of
// M=128 and M=256 MMAs), at most the tile. A group of 228 rows loads a 256-row tile but runs
// N=240 MMAs; the columns past N are never stored.
__device__ __forceinline__ int mma_cols(int nvalid, int nt) { return min(nt, (nvalid + 15) & ~15); }

// Packed expert weights are tile-major: weight block bi (R rows) and K columns TK kb .. TK kb +
// TK - 1 form one contiguous tile of R rows of 128 bytes (TK = 64 bf16 or 128 e4m3 elements),
// viewed by the tensor map as rows of a [*][TK] matrix. Coordinates (x, y) of the EK-wide K
// slice kg of block bi (K = the reduction length).
template <int EK, int TK>
__device__ __forceinline__ void weight_tile_xy(int bi, int kg, int K, int R, int& x, int& y) {
    const int k0 = kg * EK;
    x = k0 % TK;
    y = (bi * (K / TK) + k0 / TK) * R;
}

// Work table. A token tile is (group g, tile nb) of nt rows; a unit is (tile, feature block
// [, K range]), units_per_tile of them per tile, numbered tile-major, tiles in group order. The
// units are dealt to the W workers (CTAs or CTA pairs) in snake order: round i gives unit
// i*W + w to worker w on even rounds and i*W + W-1-w on odd ones, which evens out the work per
// worker when unit costs vary (skewed batches); the units of one tile (the same token rows)
// run at the same time on neighbouring workers, which share those rows in L2. (Measured: listing
// the tiles sorted by cost, largest first, made skewed batches 2-3% slower than group order.)
__device__ __forceinline__ Unit decode_unit(int u, int units_per_tile, const int32_t* tiles, const int32_t* offs,
                                            int E, int T, int nt_max) {
    const int t = tiles[u / units_per_tile];
    const int g = t >> 20;
    const int nt = group_tile(group_rows(g, E, T, offs), nt_max);
    return Unit{g, u % units_per_tile, t & 0xFFFFF, nt};
}

#ifndef SMOE_REUSE_HINT
#define SMOE_REUSE_HINT 1   // keep the weights of multi-tile groups in L2 (0: stream every weight tile)
#endif
// L2 policy of a unit's weight tiles. A group with several token tiles reads each weight tile
// once per token tile, from neighbouring workers at about the same time: those tiles are kept
// (evict-last) so that the later reads hit L2; a single-tile group's weights are read once and
// streamed (evict-first).
__device__ __forceinline__ uint64_t weight_policy(int rows, int nt, uint64_t stream_pol, uint64_t keep_pol) {
    return (SMOE_REUSE_HINT && rows > nt) ? keep_pol : stream_pol;
}

// Unit of round i for worker w of W (snake order), or -1 when it lies past the last unit.
__device__ __forceinline__ int snake_unit(int i, int w, int W, int total) {
    const int u = i * W + ((i & 1) ? W - 1 - w : w);
    return u < total ? u : -1;
}

// One warp: validate the offsets into offs[] (corrupt offsets: no routed work, the error word
// set), then list the token tiles in tiles[] (entry g << 20 | nb) in group order, the shared
// group (g = E) last or first (shared_place); the shared group's first sh_skip
// tiles are left out (they were computed before the table existed). Returns the tile count.
// Lane l owns a contiguous range of groups and one warp scan places its tiles: every CTA of the
// launch builds the same table.
enum SharedPlace { kSharedLast = 0, kSharedFirst = 1 };

__device__ int build_tile_table(const int32_t* offsets, int E, int T, int routed_rows, int nt_max, int max_tiles,
                                int32_t* offs, int32_t* tiles, int32_t* err, int shared_place, int sh_skip = 0) {
    const int lane = threadIdx.x & 31;
    bool bad = false;
    for (int i = lane; i <= E; i += 32) {
        int v = (offsets != nullptr) ? offsets[i] : 0;
        if (v < 0 || v > routed_rows) { bad = true; v = 0; }
        offs[i] = v;
    }
    __syncwarp();
    for (int i = lane; i < E; i += 32)
        if (offs[i + 1] < offs[i]) bad = true;
    if (__any_sync(0xFFFFFFFFu, bad)) {
        for (int i = lane; i <= E; i += 32) offs[i] = 0;
        if (lane == 0) record_error(err, SMOE_ERR_DEVICE);
    }
    __syncwarp();
    const int ngroups = E + 1;
    const int chunk = (ngroups + 31) / 32;
    const int o0 = min(lane * chunk, ngroups), o1 = min(o0 + chunk, ngroups);
    auto group_at = [&](int o) { return shared_place == kSharedFirst ? (o == 0 ? E : o - 1) : o; };   // position -> group
    auto skip_of = [&](int g) { return g == E ? sh_skip : 0; };
    auto tiles_of = [&](int g) {
        const int rows = group_rows(g, E, T, offs);
        const int nt = group_tile(rows, nt_max);
        return max((rows + nt - 1) / nt - skip_of(g), 0);
    };
    int local = 0;
    for (int o = o0; o < o1; ++o) local += tiles_of(group_at(o));
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int n = __shfl_up_sync(0xFFFFFFFFu, incl, off);
        if (lane >= off) incl += n;
    }
    int pos = incl - local;
    for (int o = o0; o < o1; ++o) {
        const int g = group_at(o);
        const int nblk = tiles_of(g);
        for (int nb = 0; nb < nblk; ++nb, ++pos)
            if (pos < max_tiles) tiles[pos] = (g << 20) | (nb + skip_of(g));
    }
    int n = __shfl_sync(0xFFFFFFFFu, incl, 31);
    if (n > max_tiles) {   // cannot happen for validated offsets; never read past the table
        if (lane == 0) record_error(err, SMOE_ERR_DEVICE);
        n = 0;
    }
    return n;
}

// Epilogue, part 1: drain this thread's accumulator row (one output feature, up to 256 token
// columns) into registers as packed bf16 pairs: SiLU(gate) * up for gate/up (after the SwiGLU
// clamp when lim > 0), the plain value for down. 32-column TMEM loads, one wait each.
// nch = number of 32-column chunks holding valid tokens. A thread takes the whole row (NS = 8) or,
// where two epilogue warps share a quarter of the TMEM lanes, every other chunk: its chunk i is
// accumulator chunk c0 + (8 / NS) i, and hv and cs are indexed by i.
// With F8 (e4m3 operands) the accumulators are first scaled: by rs_g * s(col) (gate, or the down
// output) and rs_u * s(col) (up), rs = this feature's weight-row scale and s(col) the activation
// scale of the column, which lane j of the warp holds in cs[i] for column 32 c + j of chunk i.
template <bool DUAL, bool F8, int NS = 8>
__device__ __forceinline__ void epi_load(uint32_t t_row, int nt_max, int nch, float lim, uint32_t (&hv)[16 * NS],
                                         float rs_g, float rs_u, const float (&cs)[NS], int c0 = 0) {
#pragma unroll
    for (int i = 0; i < NS; ++i) {
        const int c = c0 + (8 / NS) * i;
        if (c < nch) {
            uint32_t a[32], b[32];
            if (DUAL)
                tmem_ld2_x32_wait(t_row + 32 * c, t_row + nt_max + 32 * c, a, b);
            else
                tmem_ld_x32_wait(t_row + 32 * c, a);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                float v0 = __uint_as_float(a[2 * j]), v1 = __uint_as_float(a[2 * j + 1]);
                float s0 = 1.f, s1 = 1.f;
                if (F8) {
                    s0 = __shfl_sync(0xFFFFFFFFu, cs[i], 2 * j);
                    s1 = __shfl_sync(0xFFFFFFFFu, cs[i], 2 * j + 1);
                    v0 *= rs_g * s0;
                    v1 *= rs_g * s1;
                }
                if (DUAL) {
                    float u0 = __uint_as_float(b[2 * j]), u1 = __uint_as_float(b[2 * j + 1]);
                    if (F8) {
                        u0 *= rs_u * s0;
                        u1 *= rs_u * s1;
                    }
                    if (lim > 0.0f) {   // SwiGLU clamp: gate from above, up on both sides
                        v0 = fminf(v0, lim);
                        v1 = fminf(v1, lim);
                        u0 = fminf(fmaxf(u0, -lim), lim);
                        u1 = fminf(fmaxf(u1, -lim), lim);
                    }
                    v0 = silu_mul(v0, u0);
                    v1 = silu_mul(v1, u1);
                }
                hv[16 * i + j] = pack_bf16x2(v0, v1);
            }
        }
    }
}

// Epilogue, part 2: store the valid token columns of this thread's feature (after the accumulator
// has been handed back to the MMA thread); chunks as in epi_load.
template <int NS = 8>
__device__ __forceinline__ void epi_store(const uint32_t (&hv)[16 * NS], int nch, int nvalid, uint16_t* out,
                                          size_t dst0, int ld, int c0 = 0) {
#pragma unroll
    for (int i = 0; i < NS; ++i) {
        const int c = c0 + (8 / NS) * i;
        if (c < nch) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (32 * c + j < nvalid)
                    out[dst0 + (size_t)(32 * c + j) * ld] = (uint16_t)((j & 1) ? (hv[16 * i + j / 2] >> 16)
                                                                               : (hv[16 * i + j / 2] & 0xFFFFu));
        }
    }
}

// e4m3 launches: lane j loads the activation scale of columns 32 c + j of a unit (0 past its
// valid rows) for the thread's chunks c (as in epi_load); issued before the accumulator wait, so
// the loads overlap the MMAs.
template <int NS = 8>
__device__ __forceinline__ void load_col_scales(const GemmParams& p, const Unit& w, int nvalid, const int32_t* offs,
                                                int lane, float (&cs)[NS], int c0 = 0) {
    const int base = (w.g < p.E ? offs[w.g] : p.scale_shared_base) + w.nb * w.nt;
#pragma unroll
    for (int i = 0; i < NS; ++i) {
        const int col = 32 * (c0 + (8 / NS) * i) + lane;
        float v = 0.f;
        if (col < nvalid) {
            int idx = base + col;
            if (p.scale_tok != nullptr && w.g < p.E) {
                idx = p.scale_tok[idx];
                if (idx < 0 || idx >= p.T) {   // corrupt token index: never read past the scales
                    record_error(p.err, SMOE_ERR_DEVICE);
                    idx = -1;
                }
            }
            if (idx >= 0) v = p.act_scale[idx];
        }
        cs[i] = v;
    }
}

template <int MODE, int BK, bool F8>
__global__ void __launch_bounds__(kThreads, 1)
expert_gemm_kernel(const __grid_constant__ GemmMaps maps, const GemmParams p) {
    using C = GemmCfg<MODE, BK>;
    constexpr bool DUAL = C::DUAL;
    extern __shared__ uint8_t smem_raw[];
    const int S = p.stages;
    const int STAGE_B = stage_bytes(DUAL, BK, p.nt_max);
    const int ACC_COLS = DUAL ? 2 * p.nt_max : p.nt_max;
    const int NACC = (2 * ACC_COLS <= kTmemCols) ? 2 : 1;
    uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(tiles + (size_t)S * STAGE_B);
    uint64_t* empty = full + S;
    uint64_t* tfull = empty + S;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint64_t* tab_ready = drain + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tab_ready + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* ntiles_slot = reinterpret_cast<int*>(tmem_slot + 2);
    int32_t* ttab = reinterpret_cast<int32_t*>(tmem_slot + 4);     // token tiles [max_tiles]
    int32_t* offs = ttab + p.max_tiles;                              // [E+1]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = p.E;
    const int MB = p.n_out / 128;
    constexpr int EK = F8 ? 128 : BK;     // K elements per stage (128-byte rows either way)
    constexpr int TK = F8 ? 128 : 64;     // K elements per packed weight tile
    const int KB = p.K / EK / p.ksplit;   // k-blocks of one unit
    const int upt = MB * p.ksplit;        // units per token tile
    const int W = gridDim.x;

    // Shared units before the dependency wait (shared_prewait): the shared group's rows are the
    // rows of x and its weights are fixed, so its units need nothing the earlier kernels of this
    // layer compute. As many whole shared tiles as one round of CTAs holds (one unit per CTA)
    // run first, CTA b taking unit b; the table built once the offsets are known lists the
    // shared group's other tiles first, then the routed ones, dealt over all CTAs.
    const bool prewait = p.shared_prewait != 0 && p.row_token != nullptr;   // gather mode: a full producer warp
    const int nt_sh = group_tile(p.T, p.nt_max);
    const int pre_tiles = prewait ? min((p.T + nt_sh - 1) / nt_sh, W / upt) : 0;
    const int n_shared = pre_tiles * upt;   // <= W
    auto shared_unit = [&](int) { const int s = blockIdx.x; return Unit{E, s % upt, s / upt, nt_sh}; };
    auto n_shared_mine = [&]() { return blockIdx.x < (unsigned)n_shared ? 1 : 0; };

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tfull[a]), 1);
            mbar_init(smem_u32(&tempty[a]), 128);
        }
        mbar_init(smem_u32(drain), 1);
        mbar_init(smem_u32(tab_ready), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    if (warp == 1 && lane == 0) {
        tma_prefetch_desc(&maps.w);
        for (int i = 0; i < kNumTiles; ++i)
            if ((16 << i) <= p.nt_max) {
                tma_prefetch_desc(&maps.act[i]);
                tma_prefetch_desc(&maps.sh[i]);
            }
    }
    // The set-up above reads nothing an earlier kernel writes, so it overlaps that kernel's tail
    // (this CTA's shared memory rules out sharing an SM, hence TMEM, with another GEMM CTA).
    if (!prewait) {
        // everything below may read the earlier kernels' results: wait for them, then list the
        // token tiles
        pdl_wait();
        pdl_launch_dependents();
        if (warp == 2) {
            const int n = build_tile_table(p.offsets, E, p.T, p.routed_rows, p.nt_max, p.max_tiles, offs, ttab,
                                           p.err, p.shared_first != 0 ? kSharedFirst : kSharedLast);
            if (lane == 0) *ntiles_slot = n;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    // Before its first routed unit each role waits for the tile table: built above (plain
    // launch), or by the producer warp once the offsets are there (shared_prewait), which then
    // arrives on tab_ready. Returns the routed unit count.
    auto await_table = [&]() -> int {
        if (prewait) {
            if (!mbar_wait(smem_u32(tab_ready), 0u, p.err, abort_flag, true)) return 0;
            pdl_wait();
            pdl_launch_dependents();
        }
        return *ntiles_slot * upt;
    };

    // gather mode (row_token set) uses all 32 producer lanes; otherwise lane 0 alone, so the
    // stage refill path carries no warp-wide synchronisation
    const unsigned pmask = (p.row_token != nullptr) ? 0xFFFFFFFFu : 1u;
    if (warp == 0 && ((pmask >> lane) & 1u)) {
        // ---------------------------------------------------------------- TMA producer (warp 0)
        // Lane 0 waits for a free stage, arms its barrier and loads the weight tile. Activation
        // rows come either as one tile (contiguous rows) or, for routed groups in gather mode,
        // as token rows picked straight out of x by tile::gather4 loads that the 32 lanes share
        // (4 rows each; rows past the group's end repeat its last row and are never stored).
        const uint64_t pol_w = l2_policy_evict_first();
        const uint64_t pol_a = l2_policy_evict_last();
        int stage = 0;
        uint32_t phase = 0, armed = 0, armed_par = 0;
        bool ok = true;
        auto load_unit = [&](Unit w) {
            const int kb0 = (w.mb / MB) * KB;   // first k-block of this unit's K range
            w.mb %= MB;
            const int a_row = DUAL ? (w.g * MB + w.mb) * 256 : w.g * p.n_out + w.mb * 128;   // router: row-major
            const int b_row = (w.g < E ? offs[w.g] : p.shared_in_row) + w.nb * w.nt;
            const int ti = tile_index(w.nt);
            const bool gather = p.row_token != nullptr && w.g < E;
            const CUtensorMap* bm = (w.g < E) ? &maps.act[gather ? 0 : ti] : &maps.sh[ti];
            const uint32_t tx = (uint32_t)(C::A_BYTES + w.nt * BK * 2);
            const uint64_t pw = weight_policy(group_rows(w.g, E, p.T, offs), w.nt, pol_w, pol_a);
            // gather mode: this lane's chunks of 4 rows (chunk c = lane + 32 j) and their tokens
            int tok[8];
            const int nchunks = w.nt / 4;
            if (gather) {
                const int last = offs[w.g + 1] - 1;
#pragma unroll
                for (int j = 0; j < 2; ++j)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int c = lane + 32 * j;
                        const int r = min(b_row + 4 * c + i, last);
                        tok[4 * j + i] = (c < nchunks) ? p.row_token[r] : 0;
                    }
            }
            for (int kb = 0; kb < KB; ++kb) {
                if (lane == 0) ok = mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, p.err, abort_flag, true);
                ok = __shfl_sync(pmask, ok, 0);
                if (!ok) break;
                const uint32_t fb = smem_u32(&full[stage]);
                uint8_t* a_s = tiles + (size_t)stage * STAGE_B;
                const int kg = kb0 + kb;   // k-block within the whole K
                const int b_k = p.k_wrap ? (kg % p.k_wrap) : kg;
                if (lane == 0) {
                    mbar_arrive_expect_tx(fb, tx);
                    if (MODE == MODE_ROUTER) {
                        tma_load_2d(smem_u32(a_s), &maps.w, kg * BK, a_row, fb, pw);
                    } else {
                        int wx, wy;
                        weight_tile_xy<EK, TK>(w.g * MB + w.mb, kg, p.K, C::A_ROWS, wx, wy);
                        tma_load_2d(smem_u32(a_s), &maps.w, wx, wy, fb, pw);
                    }
                    if (!gather) tma_load_2d(smem_u32(a_s + C::A_BYTES), bm, b_k * EK, b_row, fb, pol_a);
                }
                __syncwarp(pmask);
                if (gather) {
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int c = lane + 32 * j;
                        if (c < nchunks)
                            tma_gather4_2d(smem_u32(a_s + C::A_BYTES + c * 4 * BK * 2), bm, b_k * EK, tok[4 * j],
                                           tok[4 * j + 1], tok[4 * j + 2], tok[4 * j + 3], fb, pol_a);
                    }
                }
                armed |= 1u << stage;
                armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                if (++stage == S) { stage = 0; phase ^= 1u; }
            }
        };
        for (int j = 0; ok && j < n_shared_mine(); ++j) load_unit(shared_unit(j));
        if (prewait) {
            // the offsets are final once the earlier kernels are done: list the routed tiles
            pdl_wait();
            pdl_launch_dependents();
            const int n = build_tile_table(p.offsets, E, p.T, p.routed_rows, p.nt_max, p.max_tiles, offs, ttab, p.err,
                                           kSharedFirst, pre_tiles);
            if (lane == 0) {
                *ntiles_slot = n;
                mbar_arrive(smem_u32(tab_ready));
            }
            __syncwarp();
        }
        const int total = *ntiles_slot * upt;
        for (int i = 0; ok && i * W < total; ++i) {
            const int u = snake_unit(i, blockIdx.x, W, total);
            if (u < 0) continue;
            load_unit(decode_unit(u, upt, ttab, offs, E, p.T, p.nt_max));
        }
        // every load issued must land before the CTA may exit
        if (lane == 0)
            for (int s = 0; s < S; ++s)
                if ((armed >> s) & 1u) mbar_wait(smem_u32(&full[s]), (armed_par >> s) & 1u, p.err, abort_flag, false);
        __syncwarp(pmask);
    } else if (warp == 1 && lane == 0) {
        // ---------------------------------------------------------------- MMA issuer
        const uint32_t idesc0 = F8 ? idesc_e4m3_f32(128, 0) : idesc_bf16_f32(128, 0);
        int stage = 0, acc = 0;
        uint32_t phase = 0, acc_phase = 0;
        bool ok = true;
        auto mma_unit = [&](const Unit& w) {
            const int n_mma = mma_cols(group_rows(w.g, E, p.T, offs) - w.nb * w.nt, w.nt);
            const uint32_t idesc = idesc0 | ((uint32_t)(n_mma >> 3) << 17);
            if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1u, p.err, abort_flag, true)) { ok = false; return; }
            tc_fence_after();
            const uint32_t d = tmem_base + (uint32_t)(acc * ACC_COLS);
            for (int kb = 0; kb < KB; ++kb) {
                if (!mbar_wait(smem_u32(&full[stage]), phase, p.err, abort_flag, true)) { ok = false; break; }
                tc_fence_after();
                const uint32_t a_s = smem_u32(tiles + (size_t)stage * STAGE_B);
                const uint32_t b_s = a_s + C::A_BYTES;
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
                    const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
                    const uint64_t bdesc = smem_desc_kmajor<C::SW>(b_s + kk * 32);
                    const uint64_t adesc = smem_desc_kmajor<C::SW>(a_s + kk * 32);
                    if (F8) umma_f8_ss(d, adesc, bdesc, idesc, accum); else umma_f16_ss(d, adesc, bdesc, idesc, accum);
                    if (DUAL) {
                        const uint64_t udesc = smem_desc_kmajor<C::SW>(a_s + C::UP_OFFSET + kk * 32);
                        if (F8)
                            umma_f8_ss(d + p.nt_max, udesc, bdesc, idesc, accum);
                        else
                            umma_f16_ss(d + p.nt_max, udesc, bdesc, idesc, accum);
                    }
                }
                umma_commit(smem_u32(&empty[stage]));
                if (++stage == S) { stage = 0; phase ^= 1u; }
            }
            if (!ok) return;
            umma_commit(smem_u32(&tfull[acc]));
            if (NACC == 2) {
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            } else {
                acc_phase ^= 1u;
            }
        };
        for (int j = 0; ok && j < n_shared_mine(); ++j) mma_unit(shared_unit(j));
        const int total = ok ? await_table() : 0;
        for (int i = 0; ok && i * W < total; ++i) {
            const int u = snake_unit(i, blockIdx.x, W, total);
            if (u < 0) continue;
            mma_unit(decode_unit(u, upt, ttab, offs, E, p.T, p.nt_max));
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
        bool ok = true;
        auto epi_unit = [&](Unit w) {
            const int kp = w.mb / MB;   // K range of this unit (partial output kp)
            w.mb %= MB;
            const int rows = group_rows(w.g, E, p.T, offs);
            const int out_base = (w.g < E ? offs[w.g] : p.shared_out_row) + w.nb * w.nt;
            const int nvalid = min(w.nt, rows - w.nb * w.nt);
            float cs[8];
            if (F8) load_col_scales(p, w, nvalid, offs, lane, cs);
            if (!mbar_wait(smem_u32(&tfull[acc]), acc_phase, p.err, abort_flag, true)) { ok = false; return; }
            tc_fence_after();
            const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * ACC_COLS);
            const int f = w.mb * 128 + row;
            const bool keep = f < p.out_valid;
            const size_t dst0 = (size_t)out_base * p.out_ld + f;
            if (MODE == MODE_ROUTER) {
                for (int c0 = 0; c0 < nvalid; c0 += 16) {
                    uint32_t g16[16];
                    tmem_ld_x16_wait(t_row + c0, g16);
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (c0 + j < nvalid && keep)
                            p.out_f32[kp * p.split_stride + dst0 + (size_t)(c0 + j) * p.out_ld] = __uint_as_float(g16[j]);
                }
                tc_fence_before();
                mbar_arrive(smem_u32(&tempty[acc]));
            } else {
                const int nch = (nvalid + 31) / 32;
                uint32_t hv[128];
                float rs_g = 1.f, rs_u = 1.f;
                if (F8) {
                    rs_g = p.w_scale[(size_t)(DUAL ? 2 * w.g : w.g) * p.n_out + f];
                    if (DUAL) rs_u = p.w_scale[(size_t)(2 * w.g + 1) * p.n_out + f];
                }
                epi_load<DUAL, F8>(t_row, p.nt_max, nch, w.g < E ? p.clamp_routed : p.clamp_shared, hv, rs_g, rs_u,
                                   cs);
                tc_fence_before();
                mbar_arrive(smem_u32(&tempty[acc]));   // accumulator free before the stores
                epi_store(hv, nch, nvalid, p.out, dst0, p.out_ld);
            }
            if (NACC == 2) {
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            } else {
                acc_phase ^= 1u;
            }
        };
        for (int j = 0; ok && j < n_shared_mine(); ++j) epi_unit(shared_unit(j));
        const int total = ok ? await_table() : 0;
        for (int i = 0; ok && i * W < total; ++i) {
            const int u = snake_unit(i, blockIdx.x, W, total);
            if (u < 0) continue;
            epi_unit(decode_unit(u, upt, ttab, offs, E, p.T, p.nt_max));
        }
    }
    if (prewait && warp == 1 && lane != 0) {   // the idle lanes of the MMA warp take part in the wait too
        pdl_wait();
        pdl_launch_dependents();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// ------------------------------------------------------------------------------------------
// CTA-pair variant (tcgen05 cta_group::2) for large token tiles.
//
// A pair of CTAs on two SMs computes one unit of 256 output features x nt tokens: each CTA
// holds the weight rows of its 128 features (for gate/up: 128 gate + 128 up rows) and half of
// the token rows (nt/2); one 256-row MMA issued by the first CTA reads both CTAs' shared memory
// and accumulates into both CTAs' TMEM (128 rows each). Per SM this moves 25-30% fewer operand
// bytes through shared memory per MMA than the single-CTA kernel, whose token tile every SM
// loads in full. Work unit = (token tile, 256-feature block), dealt to the pairs in the same
// snake order as the single-CTA kernel's units.
//
// Roles (320 threads per CTA): warp 0 loads (lane 0; all lanes issue the row gathers in gather
// mode), warp 1 lane 0 of the first CTA issues the MMAs, and warps 2-9 drain the accumulator,
// two warps per quarter of the TMEM lanes, each taking every other 32-column chunk. Two drain
// warps per SM sub-partition cut the prefill step's down GEMM by ~10% against one (the single
// drain warp's TMEM-load waits and 2-byte column stores did not hide behind the next unit's
// MMAs); four per quarter measured no faster.
//
// Signals: both CTAs' loads complete on the first CTA's stage barrier (it arms the expected
// bytes of both); the first CTA's MMA thread commits stage-free and accumulator-ready to each
// CTA's barrier; both CTAs' epilogue warps arrive on the first CTA's accumulator-free barrier.
// A cluster barrier before teardown keeps each CTA's shared memory and TMEM alive until the
// pair's MMAs are done.
// ------------------------------------------------------------------------------------------
template <int MODE, int BK, bool F8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(pair_threads<MODE>(), 1)
expert_gemm_pair_kernel(const __grid_constant__ GemmMaps maps, const GemmParams p) {
    using C = GemmCfg<MODE, BK>;
    constexpr bool DUAL = C::DUAL;
    extern __shared__ uint8_t smem_raw[];
    const int S = p.stages;
    const int STAGE_B = C::A_BYTES + (p.nt_max / 2) * BK * 2;
    const int ACC_COLS = DUAL ? 2 * p.nt_max : p.nt_max;
    const int NACC = (2 * ACC_COLS <= kTmemCols) ? 2 : 1;
    uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(tiles + (size_t)S * STAGE_B);
    uint64_t* empty = full + S;
    uint64_t* tfull = empty + S;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* ntiles_slot = reinterpret_cast<int*>(tmem_slot + 2);
    int32_t* ttab = reinterpret_cast<int32_t*>(tmem_slot + 4);     // token tiles [max_tiles]
    int32_t* offs = ttab + p.max_tiles;                              // [E+1]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int E = p.E;
    const int MB = p.n_out / 128;       // 128-row blocks of a group's weights
    const int MBP = p.n_out / 256;      // 256-feature blocks handled by a pair
    constexpr int EK = F8 ? 128 : BK;     // K elements per stage (128-byte rows either way)
    constexpr int TK = F8 ? 128 : 64;     // K elements per packed weight tile
    const int KB = p.K / EK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tfull[a]), 1);
            mbar_init(smem_u32(&tempty[a]), 2 * pair_epi_warps<MODE>());   // epilogue warps of both CTAs
        }
        mbar_init(smem_u32(drain), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish_pair();
    }
    if (warp == 1 && lane == 0) {
        tma_prefetch_desc(&maps.w);
        for (int i = 0; i < kNumTiles; ++i)
            if ((16 << i) <= p.nt_max) {
                tma_prefetch_desc(&maps.act[i]);
                tma_prefetch_desc(&maps.sh[i]);
            }
    }
    // The set-up above reads nothing an earlier kernel writes, so it overlaps that kernel's tail
    // (this CTA's shared memory rules out sharing an SM, hence TMEM, with another GEMM CTA);
    // everything below may read its results.
    pdl_wait();
    pdl_launch_dependents();
    if (warp == 2) {
        const int n = build_tile_table(p.offsets, E, p.T, p.routed_rows, p.nt_max, p.max_tiles, offs, ttab, p.err,
                                         p.shared_first != 0 ? kSharedFirst : kSharedLast);
        if (lane == 0) *ntiles_slot = n;
    }
    tc_fence_before();
    cluster_sync();   // barrier inits and TMEM allocation visible to both CTAs
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total = *ntiles_slot * MBP;   // units: (token tile, 256-feature block)

    // gather mode (row_token set): all 32 lanes of warp 0 issue row gathers; otherwise lane 0 alone
    const unsigned pmask = (p.row_token != nullptr) ? 0xFFFFFFFFu : 1u;
    if (warp == 0 && ((pmask >> lane) & 1u)) {
        // ---------------------------------------------------------------- TMA producer (both CTAs)
        // Lane 0 waits for a free stage, arms the barrier (first CTA) and loads this CTA's weight
        // tile. Its half of the token rows comes as one tile (contiguous rows), or, for routed
        // groups in gather mode, as rows picked out of x by tile::gather4 loads, lane c taking
        // rows 4c..4c+3 of the half (rows past the group's end repeat its last row; the MMA never
        // reads them).
        const uint64_t pol_w = l2_policy_evict_first();
        const uint64_t pol_a = l2_policy_evict_last();
        int stage = 0;
        uint32_t phase = 0, armed = 0, armed_par = 0;
        bool ok = true;
        for (int i = 0; ok && i * npairs < total; ++i) {
            const int u = snake_unit(i, pair, npairs, total);
            if (u < 0) continue;
            const Unit w = decode_unit(u, MBP, ttab, offs, E, p.T, p.nt_max);   // w.mb = 256-feature block
            const int a_blk = w.g * MB + 2 * w.mb + (int)rank;   // this CTA's 128-feature weight block
            // each CTA holds half of the MMA's N columns: the first CTA token rows 0..n/2-1 of the
            // tile, the second n/2..n-1 (its box of nt/2 rows may run past them; those rows are
            // never read)
            const int half = w.nt / 2;
            const int n_mma = mma_cols(group_rows(w.g, E, p.T, offs) - w.nb * w.nt, w.nt);
            const int b_row = (w.g < E ? offs[w.g] : p.shared_in_row) + w.nb * w.nt + (int)rank * (n_mma / 2);
            const int ti = tile_index(w.nt);
            const bool gather = p.row_token != nullptr && w.g < E;
            const CUtensorMap* bm = (w.g < E) ? &maps.act[gather ? 0 : ti] : &maps.sh[ti];
            const uint32_t tx = (uint32_t)(2 * (C::A_BYTES + half * BK * 2));
            const uint64_t pw = weight_policy(group_rows(w.g, E, p.T, offs), w.nt, pol_w, pol_a);
            const bool my_chunk = gather && lane < half / 4;
            int tok[4] = {0, 0, 0, 0};
            if (my_chunk) {
                const int last = offs[w.g + 1] - 1;
#pragma unroll
                for (int r = 0; r < 4; ++r) tok[r] = p.row_token[min(b_row + 4 * lane + r, last)];
            }
            for (int kb = 0; kb < KB; ++kb) {
                if (lane == 0) ok = mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, p.err, abort_flag, true);
                ok = __shfl_sync(pmask, ok, 0);
                if (!ok) break;
                const uint32_t fb_local = smem_u32(&full[stage]);
                const uint32_t fb_leader = mapa_shared(fb_local, 0);
                uint8_t* a_s = tiles + (size_t)stage * STAGE_B;
                if (lane == 0) {
                    if (rank == 0) mbar_arrive_expect_tx(fb_local, tx);
                    int wx, wy;
                    weight_tile_xy<EK, TK>(a_blk, kb, p.K, C::A_ROWS, wx, wy);
                    tma_load_2d_pair(smem_u32(a_s), &maps.w, wx, wy, fb_leader, pw);
                    if (!gather) tma_load_2d_pair(smem_u32(a_s + C::A_BYTES), bm, kb * EK, b_row, fb_leader, pol_a);
                }
                __syncwarp(pmask);
                if (my_chunk)
                    tma_gather4_2d_pair(smem_u32(a_s + C::A_BYTES + lane * 4 * BK * 2), bm, kb * EK, tok[0], tok[1],
                                        tok[2], tok[3], fb_leader, pol_a);
                armed |= 1u << stage;
                armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                if (++stage == S) { stage = 0; phase ^= 1u; }
            }
        }
        if (rank == 0 && lane == 0) {
            // both CTAs' bytes of every armed stage are counted here: wait for them to land
            for (int s = 0; s < S; ++s)
                if ((armed >> s) & 1u)
                    mbar_wait(smem_u32(&full[s]), (armed_par >> s) & 1u, p.err, abort_flag, false);
        }
        __syncwarp(pmask);
    } else if (warp == 1 && lane == 0 && rank == 0) {
        // ---------------------------------------------------------------- MMA issuer (first CTA)
        const uint32_t idesc0 = F8 ? idesc_e4m3_f32(256, 0) : idesc_bf16_f32(256, 0);
        int stage = 0, acc = 0;
        uint32_t phase = 0, acc_phase = 0;
        bool ok = true;
        for (int i = 0; ok && i * npairs < total; ++i) {
            const int u = snake_unit(i, pair, npairs, total);
            if (u < 0) continue;
            const Unit w = decode_unit(u, MBP, ttab, offs, E, p.T, p.nt_max);
            const int n_mma = mma_cols(group_rows(w.g, E, p.T, offs) - w.nb * w.nt, w.nt);
            const uint32_t idesc = idesc0 | ((uint32_t)(n_mma >> 3) << 17);
            if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1u, p.err, abort_flag, true)) break;
            tc_fence_after();
            const uint32_t d = tmem_base + (uint32_t)(acc * ACC_COLS);
            for (int kb = 0; kb < KB; ++kb) {
                if (!mbar_wait(smem_u32(&full[stage]), phase, p.err, abort_flag, true)) { ok = false; break; }
                tc_fence_after();
                const uint32_t a_s = smem_u32(tiles + (size_t)stage * STAGE_B);
                const uint32_t b_s = a_s + C::A_BYTES;
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
                    const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
                    const uint64_t bdesc = smem_desc_kmajor<C::SW>(b_s + kk * 32);
                    const uint64_t adesc = smem_desc_kmajor<C::SW>(a_s + kk * 32);
                    if (F8)
                        umma_f8_ss_pair(d, adesc, bdesc, idesc, accum);
                    else
                        umma_f16_ss_pair(d, adesc, bdesc, idesc, accum);
                    if (DUAL) {
                        const uint64_t udesc = smem_desc_kmajor<C::SW>(a_s + C::UP_OFFSET + kk * 32);
                        if (F8)
                            umma_f8_ss_pair(d + p.nt_max, udesc, bdesc, idesc, accum);
                        else
                            umma_f16_ss_pair(d + p.nt_max, udesc, bdesc, idesc, accum);
                    }
                }
                const uint32_t eb = smem_u32(&empty[stage]);
                umma_commit_pair(mapa_shared(eb, 0));
                umma_commit_pair(mapa_shared(eb, 1));
                if (++stage == S) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
            const uint32_t tb = smem_u32(&tfull[acc]);
            umma_commit_pair(mapa_shared(tb, 0));
            umma_commit_pair(mapa_shared(tb, 1));
            if (NACC == 2) {
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            } else {
                acc_phase ^= 1u;
            }
        }
        umma_commit_pair(mapa_shared(smem_u32(drain), 0));
        mbar_wait(smem_u32(drain), 0u, p.err, abort_flag, false);
    } else if (warp >= 2) {
        // ---------------------------------------------------------------- epilogue (both CTAs)
        // warp w reads TMEM lanes 32 (w % 4)..+31; with G = 1, 2 or 4 epilogue warps per lane
        // quarter, warp group c0 = (w - 2) / 4 takes the 32-column chunks c0, c0 + G, ...
        constexpr int G = pair_epi_warps<MODE>() / 4;
        static_assert(G == 1 || G == 2 || G == 4, "1, 2 or 4 epilogue warps per TMEM lane quarter");
        constexpr int NS = 8 / G;
        const int q = warp & 3;
        const int c0 = (warp - 2) >> 2;
        const int row = q * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int i = 0; i * npairs < total; ++i) {
            const int u = snake_unit(i, pair, npairs, total);
            if (u < 0) continue;
            const Unit w = decode_unit(u, MBP, ttab, offs, E, p.T, p.nt_max);
            const int rows = group_rows(w.g, E, p.T, offs);
            const int out_base = (w.g < E ? offs[w.g] : p.shared_out_row) + w.nb * w.nt;
            const int nvalid = min(w.nt, rows - w.nb * w.nt);
            float cs[NS];
            if (F8) load_col_scales<NS>(p, w, nvalid, offs, lane, cs, c0);
            if (!mbar_wait(smem_u32(&tfull[acc]), acc_phase, p.err, abort_flag, true)) break;
            tc_fence_after();
            const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * ACC_COLS);
            const int f = w.mb * 256 + (int)rank * 128 + row;
            const size_t dst0 = (size_t)out_base * p.out_ld + f;
            const int nch = (nvalid + 31) / 32;
            uint32_t hv[16 * NS];
            float rs_g = 1.f, rs_u = 1.f;
            if (F8) {
                rs_g = p.w_scale[(size_t)(DUAL ? 2 * w.g : w.g) * p.n_out + f];
                if (DUAL) rs_u = p.w_scale[(size_t)(2 * w.g + 1) * p.n_out + f];
            }
            epi_load<DUAL, F8, NS>(t_row, p.nt_max, nch, w.g < E ? p.clamp_routed : p.clamp_shared, hv, rs_g, rs_u, cs,
                                   c0);
            tc_fence_before();
            __syncwarp();
            // accumulator free: every lane's TMEM loads have completed (tcgen05.wait::ld), so the
            // arrive needs no release; a release would first wait for the previous unit's stores
            if (lane == 0) mbar_arrive_cluster_relaxed(mapa_shared(smem_u32(&tempty[acc]), 0));
            epi_store<NS>(hv, nch, nvalid, p.out, dst0, p.out_ld, c0);
            if (NACC == 2) {
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            } else {
                acc_phase ^= 1u;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag) __nanosleep(100000);   // give loads still in flight after a timeout time to land
    cluster_sync();   // the peer's shared memory and TMEM stay alive until the pair's MMAs are done
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kTmemCols);
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

// 2D bf16 tensor [rows][cols] row-major; box = BK columns (2*BK bytes, swizzled) x box_rows.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows, int bk) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)bk, box_rows};
    cuuint32_t estr[2] = {1, 1};
    const CUtensorMapSwizzle sw = bk == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                           : (bk == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2D e4m3 tensor [rows][cols] (one byte per element) row-major; box = 128 columns (128 bytes,
// swizzled) x box_rows.
bool make_map_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols};
    cuuint32_t box[2] = {128, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A bf16 (bk-wide boxes) or, with u8, an e4m3 (128-wide boxes) activation map.
bool make_any_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows, int bk, bool u8) {
    return u8 ? make_map_u8(m, base, rows, cols, box_rows) : make_map(m, base, rows, cols, box_rows, bk);
}

// Activation maps for every token tile up to nt_max (larger entries repeat a valid map, unused).
bool make_act_maps(CUtensorMap* maps, const void* base, uint64_t rows, uint64_t cols, int nt_max, int bk,
                   bool u8 = false) {
    for (int i = 0; i < kNumTiles; ++i) {
        const int nt = 16 << i;
        if (nt <= nt_max) {
            if (!make_any_map(&maps[i], base, rows, cols, nt, bk, u8)) return false;
        } else {
            maps[i] = maps[i - 1];
        }
    }
    return true;
}

int max_dynamic_smem() {
    static int v = 0;
    if (v == 0) {
        int dev = 0, n = 0;
        if (cudaGetDevice(&dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) == cudaSuccess && n > 0)
            v = n;
        else
            v = 227 * 1024;
    }
    return v;
}

template <int MODE, bool F8 = false>
cudaError_t run_gemm(const GemmMaps& maps, GemmParams p, int grid, cudaStream_t s) {
    constexpr int BK = SMOE_GEMM_BK;
    constexpr bool DUAL = MODE == MODE_GATEUP;
    const int sb = stage_bytes(DUAL, BK, p.nt_max);
    p.max_tiles = max_token_tiles(p.E, p.routed_rows, p.T, p.nt_max);
    const size_t fixed = gemm_smem_bytes(0, sb, p.E, p.max_tiles) + 2 * sizeof(uint64_t) * kMaxStages;
    if (fixed >= (size_t)max_dynamic_smem()) return cudaErrorInvalidConfiguration;
    int stages = (int)((max_dynamic_smem() - fixed) / sb);
    if (stages > kMaxStages) stages = kMaxStages;
    if (stages < 2) return cudaErrorInvalidConfiguration;
    p.stages = stages;
    const size_t smem = gemm_smem_bytes(stages, sb, p.E, p.max_tiles);
    cudaError_t e = cudaFuncSetAttribute(expert_gemm_kernel<MODE, BK, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    {
        LaunchTimer lt(MODE == MODE_GATEUP ? K_EXPERT_GATEUP : (MODE == MODE_DOWN ? K_EXPERT_DOWN : K_ROUTER_GEMM), s);
        return launch_pdl(expert_gemm_kernel<MODE, BK, F8>, dim3(grid), dim3(kThreads), smem, s, maps, p);
    }
}

// Activation maps for CTA pairs: each CTA loads half of a token tile (box rows 8 << i).
bool make_half_act_maps(CUtensorMap* maps, const void* base, uint64_t rows, uint64_t cols, int nt_max, int bk,
                        bool u8 = false) {
    for (int i = 0; i < kNumTiles; ++i) {
        const int nt = 16 << i;
        if (nt <= nt_max) {
            if (!make_any_map(&maps[i], base, rows, cols, nt / 2, bk, u8)) return false;
        } else {
            maps[i] = maps[i - 1];
        }
    }
    return true;
}

template <int MODE, bool F8 = false>
cudaError_t run_gemm_pair(const GemmMaps& maps, GemmParams p, int num_sms, cudaStream_t s) {
    constexpr int BK = SMOE_GEMM_BK;
    constexpr bool DUAL = MODE == MODE_GATEUP;
    const int sb = (DUAL ? 256 : 128) * BK * 2 + (p.nt_max / 2) * BK * 2;
    p.max_tiles = max_token_tiles(p.E, p.routed_rows, p.T, p.nt_max);
    const size_t fixed = gemm_smem_bytes(0, sb, p.E, p.max_tiles) + 2 * sizeof(uint64_t) * kMaxStages;
    if (fixed >= (size_t)max_dynamic_smem()) return cudaErrorInvalidConfiguration;
    int stages = (int)((max_dynamic_smem() - fixed) / sb);
    if (stages > kMaxStages) stages = kMaxStages;
    if (stages < 2) return cudaErrorInvalidConfiguration;
    p.stages = stages;
    const size_t smem = gemm_smem_bytes(stages, sb, p.E, p.max_tiles);
    auto kern = expert_gemm_pair_kernel<MODE, BK, F8>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // pairs resident at once (a GPC with an odd number of free SMs cannot host a pair there)
    static int max_clusters_by[2][3] = {{0, 0, 0}, {0, 0, 0}};
    int* max_clusters = max_clusters_by[F8 ? 1 : 0];
    if (max_clusters[MODE] == 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(num_sms & ~1);
        cfg.blockDim = dim3(pair_threads<MODE>());
        cfg.dynamicSmemBytes = smem;
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
        if (e != cudaSuccess) return e;
        max_clusters[MODE] = n > 0 ? n : 1;
    }
    const int pairs = std::min(num_sms / 2, max_clusters[MODE]);
    {
        LaunchTimer lt(MODE == MODE_GATEUP ? K_EXPERT_GATEUP : K_EXPERT_DOWN, s);
        return launch_pdl(kern, dim3(2 * pairs), dim3(pair_threads<MODE>()), smem, s, maps, p);
    }
}

}  // namespace

#ifndef SMOE_SHARED_FIRST
#define SMOE_SHARED_FIRST 1   // small-tile gate/up launches list the shared expert's tiles first
#endif

// Largest token tile of a launch: the smallest power of two >= 1.25 x the mean rows per routed
// expert, 16..256. Groups with fewer rows use smaller tiles inside the kernel.
#ifndef SMOE_TILE_FACTOR
#define SMOE_TILE_FACTOR 1.25
#endif
int choose_token_tile(const smoe_config_t& c, int64_t T) {
    const double mean = (double)T * c.top_k / c.n_experts;
    int nt = 16;
    while (nt < SMOE_MAX_TOKEN_TILE && nt < SMOE_TILE_FACTOR * mean) nt *= 2;
    return nt;
}

// Shared units before the wait only when all of them fit in one round of CTAs (decode-sized
// batches): with more (the MTP batch's 16 tiles), the GEMM launched early competes with the
// top-k kernel's CTAs for the SMs and the routing takes longer than the overlap saves.
bool shared_prewait_fits(const smoe_config_t& c, int64_t T, int num_sms) {
    const int nt = choose_token_tile(c, T);
    int nt_sh = 16;
    while (nt_sh < T && nt_sh < nt) nt_sh *= 2;
    return (T + nt_sh - 1) / nt_sh * (c.inter / 128) <= num_sms;
}

size_t packed_gateup_bytes(const smoe_config_t& c) {
    return (size_t)(c.n_experts + 1) * 2 * c.inter * c.hidden * 2;
}
size_t packed_down_bytes(const smoe_config_t& c) { return (size_t)(c.n_experts + 1) * c.hidden * c.inter * 2; }

cudaError_t launch_expert_ffn(const smoe_config_t& c, const uint16_t* x, const uint16_t* x_perm,
                              const int32_t* row_token, const int32_t* offsets, int64_t T, const void* packed,
                              uint16_t* y, uint16_t* h, int32_t* err, int num_sms, cudaStream_t s,
                              bool shared_prewait) {
    constexpr int BK = SMOE_GEMM_BK;
    const int E = c.n_experts, H = c.hidden, I = c.inter, k = c.top_k;
    const int64_t routed = T * k;
    const int nt = choose_token_tile(c, T);
    const uint8_t* wgu = static_cast<const uint8_t*>(packed);
    const uint8_t* wdn = wgu + packed_gateup_bytes(c);

    GemmMaps m1, m2;
    const bool gather = x_perm == nullptr;
    // CTA pairs for large token tiles (each pair handles 256 output features)
    const bool pairs = nt >= kPairMinTile && I % 256 == 0 && H % 256 == 0;
    auto act_maps = [&](CUtensorMap* maps, const void* base, uint64_t rows, uint64_t cols) {
        return pairs ? make_half_act_maps(maps, base, rows, cols, nt, BK) : make_act_maps(maps, base, rows, cols, nt, BK);
    };
    bool ok_act = gather ? make_map(&m1.act[0], x, (uint64_t)T, H, 1, BK) : act_maps(m1.act, x_perm, (uint64_t)routed, H);
    if (gather)
        for (int i = 1; i < kNumTiles; ++i) m1.act[i] = m1.act[0];
    // packed weights, tile-major: viewed as [rows][64] with 256-row (gate/up) / 128-row (down) tiles
    if (!ok_act || !make_map(&m1.w, wgu, (uint64_t)(E + 1) * 2 * I * (H / 64), 64, 256, BK) ||
        !act_maps(m1.sh, x, (uint64_t)T, H) ||
        !make_map(&m2.w, wdn, (uint64_t)(E + 1) * H * (I / 64), 64, 128, BK) ||
        !act_maps(m2.act, h, (uint64_t)(routed + T), I))
        return cudaErrorNotSupported;
    for (int i = 0; i < kNumTiles; ++i) m2.sh[i] = m2.act[i];

    GemmParams p1{offsets, E, (int)T, (int)routed, H, I, 0, (int)routed, nt, 0, 0, I, I, gather ? row_token : nullptr,
                  c.swiglu_limit, c.swiglu_limit_shared, 1, 0, h, nullptr, err};
    p1.shared_first = gather && !pairs && SMOE_SHARED_FIRST ? 1 : 0;
    p1.shared_prewait = gather && !pairs && shared_prewait && shared_prewait_fits(c, T, num_sms) ? 1 : 0;
    cudaError_t e = pairs ? run_gemm_pair<MODE_GATEUP>(m1, p1, num_sms, s) : run_gemm<MODE_GATEUP>(m1, p1, num_sms, s);
    if (e != cudaSuccess) return e;
    GemmParams p2{offsets, E, (int)T, (int)routed, I, H, (int)routed, (int)routed, nt, 0, 0, H, H, nullptr, 0.f, 0.f, 1,
                  0, y, nullptr, err};
    e = pairs ? run_gemm_pair<MODE_DOWN>(m2, p2, num_sms, s) : run_gemm<MODE_DOWN>(m2, p2, num_sms, s);
    if (e == cudaSuccess) launches_add(2);
    return e;
}

cudaError_t launch_expert_ffn_fp8(const smoe_config_t& c, const uint8_t* x_q, const uint8_t* x_q_perm,
                                  const float* s_x, const int32_t* row_token, const int32_t* offsets, int64_t T,
                                  const void* packed_fp8, uint16_t* y, uint16_t* h, uint8_t* h_q, float* s_h,
                                  int32_t* err, int num_sms, cudaStream_t s) {
    constexpr int BK = SMOE_GEMM_BK;
    const int E = c.n_experts, H = c.hidden, I = c.inter, k = c.top_k;
    const int64_t routed = T * k;
    const int nt = choose_token_tile(c, T);
    const Fp8Layout L = fp8_layout(c);
    const uint8_t* pk = static_cast<const uint8_t*>(packed_fp8);

    GemmMaps m1, m2;
    const bool gather = x_q_perm == nullptr;
    const bool pairs = nt >= kPairMinTile && I % 256 == 0 && H % 256 == 0;
    auto act_maps = [&](CUtensorMap* maps, const void* base, uint64_t rows, uint64_t cols) {
        return pairs ? make_half_act_maps(maps, base, rows, cols, nt, BK, true)
                     : make_act_maps(maps, base, rows, cols, nt, BK, true);
    };
    bool ok_act = gather ? make_map_u8(&m1.act[0], x_q, (uint64_t)T, H, 1) : act_maps(m1.act, x_q_perm, (uint64_t)routed, H);
    if (gather)
        for (int i = 1; i < kNumTiles; ++i) m1.act[i] = m1.act[0];
    // packed codes, tile-major: viewed as [rows][128] with 256-row (gate/up) / 128-row (down) tiles
    if (!ok_act || !make_map_u8(&m1.w, pk + L.gateup, (uint64_t)(E + 1) * 2 * I * (H / 128), 128, 256) ||
        !act_maps(m1.sh, x_q, (uint64_t)T, H) ||
        !make_map_u8(&m2.w, pk + L.down, (uint64_t)(E + 1) * H * (I / 128), 128, 128) ||
        !act_maps(m2.act, h_q, (uint64_t)(routed + T), I))
        return cudaErrorNotSupported;
    for (int i = 0; i < kNumTiles; ++i) m2.sh[i] = m2.act[i];

    GemmParams p1{offsets, E, (int)T, (int)routed, H, I, 0, (int)routed, nt, 0, 0, I, I, gather ? row_token : nullptr,
                  c.swiglu_limit, c.swiglu_limit_shared, 1, 0, h, nullptr, err};
    p1.w_scale = reinterpret_cast<const float*>(pk + L.gateup_scale);
    p1.act_scale = s_x;
    p1.scale_tok = row_token;
    p1.scale_shared_base = 0;
    p1.shared_first = gather && !pairs && SMOE_SHARED_FIRST ? 1 : 0;
    cudaError_t e = pairs ? run_gemm_pair<MODE_GATEUP, true>(m1, p1, num_sms, s)
                          : run_gemm<MODE_GATEUP, true>(m1, p1, num_sms, s);
    if (e != cudaSuccess) return e;
    e = launch_quantize_rows(h, routed + T, I, h_q, s_h, K_QUANT_H, s);
    if (e != cudaSuccess) return e;
    GemmParams p2{offsets, E, (int)T, (int)routed, I, H, (int)routed, (int)routed, nt, 0, 0, H, H, nullptr, 0.f, 0.f, 1,
                  0, y, nullptr, err};
    p2.w_scale = reinterpret_cast<const float*>(pk + L.down_scale);
    p2.act_scale = s_h;
    p2.scale_tok = nullptr;
    p2.scale_shared_base = (int)routed;
    e = pairs ? run_gemm_pair<MODE_DOWN, true>(m2, p2, num_sms, s) : run_gemm<MODE_DOWN, true>(m2, p2, num_sms, s);
    if (e == cudaSuccess) launches_add(2);
    return e;
}

// Router logits on the tensor cores: partial[p][T][E] = x [T][H] . W_p^T for the three bf16
// pieces p = hi, mid, lo of W_r; w_split [e_pad][3H] holds the pieces of each fp32 router row
// side by side (rows >= E are zero). One group of T rows; each unit covers one piece's K range
// (x's K coordinate wraps), so the three partials are summed later in a fixed order.
cudaError_t launch_router_gemm(const uint16_t* x, int64_t T, int H, const uint16_t* w_split, int e_pad, int E,
                               float* logits, int nt, int ksplit, int num_sms, cudaStream_t s) {
    constexpr int BK = SMOE_GEMM_BK;
    GemmMaps m;
    if (!make_map(&m.w, w_split, (uint64_t)e_pad, (uint64_t)3 * H, 128, BK) ||
        !make_act_maps(m.sh, x, (uint64_t)T, H, nt, BK))
        return cudaErrorNotSupported;
    for (int i = 0; i < kNumTiles; ++i) m.act[i] = m.sh[i];
    GemmParams p{nullptr, 0, (int)T, 0, 3 * H, e_pad, 0, 0, nt, 0, H / BK, E, E, nullptr, 0.f, 0.f, ksplit, (size_t)T * E,
                 nullptr, logits, nullptr};
    return run_gemm<MODE_ROUTER>(m, p, num_sms, s);
}

}  // namespace smoe
