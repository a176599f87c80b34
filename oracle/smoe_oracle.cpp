// fp64 CPU oracle for one sparse MoE FFN layer of Step 3.5 Flash: a plain C++17 program.
//
// TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline and
// reference legs load this library (through oracle/cpp.py). It shares no code with the CUDA
// library: no headers, helpers, tables or pre/post-processing; neither includes the other.
//
// Plain loops in fp64, no BLAS, no intermediate rounding: every dot product is a sequential sum
// in index order (compiled with -ffp-contract=off, so a*b+c is a multiply then an add). Work is
// spread over std::thread workers, each output element computed by exactly one thread, so the
// results do not depend on the thread count. Top-k is a full std::sort of the experts under the
// tie rule.
//
// What it computes (the pages, by title and section):
//   * Step-3.5-Flash model card (llm-atlas), raw config fields: hidden_size 4096,
//     moe_num_experts 288, moe_top_k 8, moe_intermediate_size 1280, share_expert_dim 1280,
//     norm_expert_weight true, moe_router_activation sigmoid, moe_router_scaling_factor 3,
//     use_moe_router_bias true, need_fp32_gate true.
//   * Step 3.5 Flash summary (hyper.ai), "方法": every token goes to 8 of the 288 routed experts
//     and to the one shared expert.
//   * Step 3.5 Flash (paperlayer.ai summary), §4.1.2: the router bias is the loss-free
//     balancing device, so it steers selection; §B: the expert is a SwiGLU with gate and up
//     projections; §4.1.3 and §B: activation clipping of the deepest layers.
//
// Readings where the pages are silent (the same as the numpy restatement in oracle/moe.py):
//   1. bias for selection only; weights from the unbiased sigmoid scores;
//   2. weights: the selected scores normalised to sum 1, then times the scale (3);
//   3. expert F(x) = W_d (SiLU(W_g x) * (W_u x)), SiLU(z) = z / (1 + e^-z);
//   4. shared expert added with weight 1;
//   5. top-k order: biased score descending, then larger raw logit, then smaller expert index;
//   6. near tie: k-th minus (k+1)-th biased score below 1e-5; every selection in that band is
//      correct (so_valid_selections enumerates them);
//   7. output = FFN output only (no residual, no norm);
//   8. clamp with limit L > 0: gate min(g, L), up clamp(u, -L, L), before SiLU(g) * u.
//
// All arrays are row-major, caller-owned host memory. Functions return 0 on success and a
// negative code on bad arguments or data (-1 bad argument, -2 expert id out of range, -3 the
// expert callback failed).

#include <algorithm>
#include <chrono>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <functional>
#include <numeric>
#include <thread>
#include <vector>

namespace {

int g_threads = 0;   // 0: std::thread::hardware_concurrency()

int thread_count() {
    int n = g_threads > 0 ? g_threads : static_cast<int>(std::thread::hardware_concurrency());
    return n > 0 ? n : 1;
}

// body(i) for every i in [0, n), split into contiguous blocks over the worker threads.
void parallel_for(int64_t n, const std::function<void(int64_t)>& body) {
    const int64_t nt = std::min<int64_t>(thread_count(), n);
    if (nt <= 1) {
        for (int64_t i = 0; i < n; ++i) body(i);
        return;
    }
    std::vector<std::thread> pool;
    for (int64_t p = 0; p < nt; ++p) {
        const int64_t lo = n * p / nt, hi = n * (p + 1) / nt;
        pool.emplace_back([lo, hi, &body] {
            for (int64_t i = lo; i < hi; ++i) body(i);
        });
    }
    for (auto& th : pool) th.join();
}

// sum_i a[i] * b[i], added in index order.
double dot(const double* a, const double* b, int64_t n) {
    double acc = 0.0;
    for (int64_t i = 0; i < n; ++i) acc += a[i] * b[i];
    return acc;
}

double sigmoid(double z) { return 1.0 / (1.0 + std::exp(-z)); }

double silu(double z) { return z / (1.0 + std::exp(-z)); }

// Biased-score order of the experts of one token (readings 1 and 5).
std::vector<int32_t> ranked_experts(const double* bhat, const double* logit, int32_t E) {
    std::vector<int32_t> order(E);
    std::iota(order.begin(), order.end(), 0);
    std::sort(order.begin(), order.end(), [&](int32_t a, int32_t b) {
        if (bhat[a] != bhat[b]) return bhat[a] > bhat[b];
        if (logit[a] != logit[b]) return logit[a] > logit[b];
        return a < b;
    });
    return order;
}

// SwiGLU hidden of n rows: hid[r][i] = SiLU(g) * u with g = W_g[i] . X[r], u = W_u[i] . X[r],
// clamped first when limit > 0 (reading 8).
void swiglu_hidden_rows(const double* X, int64_t n, int64_t H, const double* Wg, const double* Wu, int64_t I,
                        double limit, double* hid) {
    // feature-major order so one thread's consecutive items reuse a weight row
    parallel_for(n * I, [&](int64_t q) {
        const int64_t i = q / n, r = q % n;
        double g = dot(Wg + i * H, X + r * H, H);
        double u = dot(Wu + i * H, X + r * H, H);
        if (limit > 0.0) {
            g = std::min(g, limit);
            u = std::min(std::max(u, -limit), limit);
        }
        hid[r * I + i] = silu(g) * u;
    });
}

// F(x) = W_d hid for n rows.
void swiglu_ffn_rows(const double* X, int64_t n, int64_t H, const double* Wg, const double* Wu, const double* Wd,
                     int64_t I, double limit, double* Y) {
    std::vector<double> hid(static_cast<size_t>(n * I));
    swiglu_hidden_rows(X, n, H, Wg, Wu, I, limit, hid.data());
    parallel_for(n * H, [&](int64_t q) {
        const int64_t o = q / n, r = q % n;
        Y[r * H + o] = dot(Wd + o * I, hid.data() + r * I, I);
    });
}

}  // namespace

extern "C" {

// Expert weights on demand: fills fp64 W_g [I][H], W_u [I][H], W_d [H][I] of expert e (e == E:
// the shared expert); the pointers must stay valid until the next call. Returns 0 on success.
typedef int (*so_expert_fn)(void* ctx, int32_t e, const double** wg, const double** wu, const double** wd);

void so_set_threads(int32_t n) { g_threads = n; }

int32_t so_threads(void) { return thread_count(); }

// bf16 bit patterns -> fp64, exactly: the bf16 bits are the upper half of an fp32.
void so_bf16_to_f64(const uint16_t* in, int64_t n, double* out) {
    const int64_t block = 1 << 16;
    parallel_for((n + block - 1) / block, [&](int64_t b) {
        for (int64_t i = b * block; i < std::min(n, (b + 1) * block); ++i) {
            const uint32_t bits = static_cast<uint32_t>(in[i]) << 16;
            float f;
            std::memcpy(&f, &bits, sizeof f);
            out[i] = static_cast<double>(f);
        }
    });
}

// fp32 -> fp64, exactly.
void so_f32_to_f64(const float* in, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = static_cast<double>(in[i]);
}

void so_sigmoid(const double* z, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = sigmoid(z[i]);
}

void so_silu(const double* z, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = silu(z[i]);
}

// Router logits (the fp32 gate, model card need_fp32_gate): L[t][e] = sum_h x[t][h] W_r[e][h].
int so_router_logits(const double* x, int64_t T, int64_t H, const double* w_router, int64_t E, double* L) {
    if (T < 0 || H <= 0 || E <= 0) return -1;
    parallel_for(T * E, [&](int64_t q) {
        const int64_t t = q / E, e = q % E;
        L[q] = dot(x + t * H, w_router + e * H, H);
    });
    return 0;
}

// Top-k of each token by biased score under the tie rule (reading 5); gap[t] = k-th minus
// (k+1)-th biased score (+inf when E == k).
int so_select_topk(const double* bhat, const double* logits, int64_t T, int32_t E, int32_t k, int32_t* idx,
                   double* gap) {
    if (T < 0 || E <= 0 || k <= 0 || k > E) return -1;
    parallel_for(T, [&](int64_t t) {
        const std::vector<int32_t> order = ranked_experts(bhat + t * E, logits + t * E, E);
        for (int32_t j = 0; j < k; ++j) idx[t * k + j] = order[j];
        gap[t] = E > k ? bhat[t * E + order[k - 1]] - bhat[t * E + order[k]] : INFINITY;
    });
    return 0;
}

// Weights of n tokens from their k selected unbiased scores (readings 1, 2; model card
// norm_expert_weight, moe_router_scaling_factor): w_j = scale * (s_j / sum_j' s_j'), the sum taken
// in slot order.
int so_normalise(const double* s_sel, int64_t n, int32_t k, double scale, double* w) {
    if (n < 0 || k <= 0) return -1;
    for (int64_t t = 0; t < n; ++t) {
        double sum = 0.0;
        for (int32_t j = 0; j < k; ++j) sum += s_sel[t * k + j];
        for (int32_t j = 0; j < k; ++j) w[t * k + j] = scale * (s_sel[t * k + j] / sum);
    }
    return 0;
}

// The router (model card moe_router_activation sigmoid, use_moe_router_bias, moe_top_k,
// norm_expert_weight, moe_router_scaling_factor): L = x W_r^T; s = sigmoid(L); bhat = s + bias;
// top-k of bhat; w_j = scale * (s_j / sum of the k selected s).
int so_route(const double* x, int64_t T, int64_t H, const double* w_router, int32_t E, const double* bias,
             int32_t k, double scale, double* L, double* s, double* bhat, int32_t* idx, double* w, double* gap) {
    if (so_router_logits(x, T, H, w_router, E, L) != 0) return -1;
    for (int64_t q = 0; q < T * E; ++q) {
        s[q] = sigmoid(L[q]);
        bhat[q] = s[q] + bias[q % E];
    }
    if (so_select_topk(bhat, L, T, E, k, idx, gap) != 0) return -1;
    std::vector<double> s_sel(static_cast<size_t>(T * k));
    for (int64_t t = 0; t < T; ++t)
        for (int32_t j = 0; j < k; ++j) s_sel[t * k + j] = s[t * E + idx[t * k + j]];
    return so_normalise(s_sel.data(), T, k, scale, w);
}

// Every k-subset S (ascending expert ids) with min over S of bhat >= max outside S of bhat - eps.
// Writes up to max_sets of them to sets [max_sets][k]; returns how many exist (or -1).
int64_t so_valid_selections(const double* bhat, int32_t E, int32_t k, double eps, int32_t* sets, int64_t max_sets) {
    if (E <= 0 || k <= 0 || k > E) return -1;
    if (E == k) {
        if (max_sets > 0)
            for (int32_t j = 0; j < k; ++j) sets[j] = j;
        return 1;
    }
    std::vector<double> v(bhat, bhat + E);
    std::sort(v.begin(), v.end(), std::greater<double>());
    std::vector<int32_t> must, cand;
    for (int32_t e = 0; e < E; ++e) {
        if (bhat[e] > v[k] + eps)
            must.push_back(e);
        else if (bhat[e] >= v[k - 1] - eps)
            cand.push_back(e);
    }
    const int32_t extra = k - static_cast<int32_t>(must.size());
    if (extra < 0) return 0;
    int64_t found = 0;
    std::vector<int32_t> pick;   // positions in cand of the current combination
    std::function<void(size_t)> visit = [&](size_t from) {
        if (static_cast<int32_t>(pick.size()) == extra) {
            std::vector<char> in(E, 0);
            for (int32_t e : must) in[e] = 1;
            for (int32_t p : pick) in[cand[p]] = 1;
            double lo = INFINITY, hi = -INFINITY;
            for (int32_t e = 0; e < E; ++e) {
                if (in[e]) lo = std::min(lo, bhat[e]);
                else hi = std::max(hi, bhat[e]);
            }
            if (lo >= hi - eps) {
                if (found < max_sets) {
                    int32_t j = 0;
                    for (int32_t e = 0; e < E; ++e)
                        if (in[e]) sets[found * k + j++] = e;
                }
                ++found;
            }
            return;
        }
        for (size_t p = from; p < cand.size(); ++p) {
            pick.push_back(static_cast<int32_t>(p));
            visit(p + 1);
            pick.pop_back();
        }
    };
    visit(0);
    return found;
}

// Token -> expert dispatch: entry p = t*k + j goes to row r, rows ordered by expert, then token,
// then slot (a counting sort). counts [E], offsets [E+1] (exclusive scan), perm_row [T*k]
// (entry -> row), row_token [T*k] (row -> token).
int so_permute(const int32_t* idx, int64_t T, int32_t k, int32_t E, int32_t* counts, int32_t* offsets,
               int32_t* perm_row, int32_t* row_token) {
    if (T < 0 || k <= 0 || E <= 0) return -1;
    for (int32_t e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t p = 0; p < T * k; ++p) {
        if (idx[p] < 0 || idx[p] >= E) return -2;
        counts[idx[p]] += 1;
    }
    offsets[0] = 0;
    for (int32_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    std::vector<int32_t> next(offsets, offsets + E);
    for (int64_t t = 0; t < T; ++t)
        for (int32_t j = 0; j < k; ++j) {
            const int32_t r = next[idx[t * k + j]]++;
            perm_row[t * k + j] = r;
            row_token[r] = static_cast<int32_t>(t);
        }
    return 0;
}

// hid = SiLU(X W_g^T) * (X W_u^T) for n rows of X [n][H] (clamped when limit > 0).
int so_swiglu_hidden(const double* X, int64_t n, int64_t H, const double* Wg, const double* Wu, int64_t I,
                     double limit, double* hid) {
    if (n < 0 || H <= 0 || I <= 0) return -1;
    swiglu_hidden_rows(X, n, H, Wg, Wu, I, limit, hid);
    return 0;
}

// Y = F(X) for n rows, F the SwiGLU expert (reading 3, clamp reading 8).
int so_swiglu_ffn(const double* X, int64_t n, int64_t H, const double* Wg, const double* Wu, const double* Wd,
                  int64_t I, double limit, double* Y) {
    if (n < 0 || H <= 0 || I <= 0) return -1;
    swiglu_ffn_rows(X, n, H, Wg, Wu, Wd, I, limit, Y);
    return 0;
}

// The layer: out[t] = F_shared(x_t) + sum over the selected experts e of w[t, e] F_e(x_t).
//   dense == 0 (sparse mode): only the selected experts are computed;
//   dense != 0 (dense-masked): every routed expert is computed for every token and multiplied by
//   its 0/1 selection mask times its weight.
// Both add the terms in the same order (shared, then experts by ascending id), and a masked term
// is an exact zero, so the two modes agree bit for bit on finite values.
int so_moe(int32_t dense, const double* x, int64_t T, int64_t H, int32_t E, int32_t k, int64_t I,
           const int32_t* idx, const double* w, so_expert_fn fetch, void* ctx, double limit, double limit_shared,
           double* out) {
    if (T < 0 || H <= 0 || E <= 0 || k <= 0 || I <= 0) return -1;
    for (int64_t p = 0; p < T * k; ++p)
        if (idx[p] < 0 || idx[p] >= E) return -2;
    const double *wg, *wu, *wd;
    if (fetch(ctx, E, &wg, &wu, &wd) != 0) return -3;
    swiglu_ffn_rows(x, T, H, wg, wu, wd, I, limit_shared, out);
    std::vector<double> Y, X;
    for (int32_t e = 0; e < E; ++e) {
        // (token, weight) pairs of expert e; in dense mode every token, weight 0 where unselected
        std::vector<int64_t> tok;
        std::vector<double> wt;
        for (int64_t t = 0; t < T; ++t) {
            double m = 0.0;
            bool sel = false;
            for (int32_t j = 0; j < k; ++j)
                if (idx[t * k + j] == e) {
                    m = w[t * k + j];
                    sel = true;
                }
            if (sel || dense) {
                tok.push_back(t);
                wt.push_back(sel ? m : 0.0);
            }
        }
        if (tok.empty()) continue;
        if (fetch(ctx, e, &wg, &wu, &wd) != 0) return -3;
        const int64_t n = static_cast<int64_t>(tok.size());
        X.resize(static_cast<size_t>(n * H));
        for (int64_t r = 0; r < n; ++r) std::memcpy(&X[r * H], x + tok[r] * H, sizeof(double) * H);
        Y.resize(static_cast<size_t>(n * H));
        swiglu_ffn_rows(X.data(), n, H, wg, wu, wd, I, limit, Y.data());
        for (int64_t r = 0; r < n; ++r)
            for (int64_t c = 0; c < H; ++c) out[tok[r] * H + c] += wt[r] * Y[r * H + c];
    }
    return 0;
}

// The output row of one token for a given selection sel[0..n_sel) (used for near-tie tokens):
// weights from the token's unbiased scores s_t [E] as in so_route, terms added in sel's order
// after the shared expert.
int so_moe_given_selection(const double* x_t, const double* s_t, const int32_t* sel, int32_t n_sel, int64_t H,
                           int32_t E, int64_t I, double scale, so_expert_fn fetch, void* ctx, double limit,
                           double limit_shared, double* out) {
    if (n_sel <= 0 || H <= 0 || I <= 0) return -1;
    for (int32_t j = 0; j < n_sel; ++j)
        if (sel[j] < 0 || sel[j] >= E) return -2;
    std::vector<double> s_sel(static_cast<size_t>(n_sel)), w_sel(static_cast<size_t>(n_sel));
    for (int32_t j = 0; j < n_sel; ++j) s_sel[j] = s_t[sel[j]];
    so_normalise(s_sel.data(), 1, n_sel, scale, w_sel.data());
    const double *wg, *wu, *wd;
    if (fetch(ctx, E, &wg, &wu, &wd) != 0) return -3;
    swiglu_ffn_rows(x_t, 1, H, wg, wu, wd, I, limit_shared, out);
    std::vector<double> y(static_cast<size_t>(H));
    for (int32_t j = 0; j < n_sel; ++j) {
        if (fetch(ctx, sel[j], &wg, &wu, &wd) != 0) return -3;
        swiglu_ffn_rows(x_t, 1, H, wg, wu, wd, I, limit, y.data());
        for (int64_t c = 0; c < H; ++c) out[c] += w_sel[j] * y[c];
    }
    return 0;
}

// Combine: out[t] = y[T*k + t] + sum_j w[t][j] y[perm_row[t*k + j]] (y: the T*k routed rows in
// expert order, then the T shared rows), terms added in slot order.
int so_combine(const double* y, const int32_t* perm_row, const double* w, int64_t T, int32_t k, int64_t H,
               double* out) {
    if (T < 0 || k <= 0 || H <= 0) return -1;
    for (int64_t p = 0; p < T * k; ++p)
        if (perm_row[p] < 0 || perm_row[p] >= T * k) return -2;
    parallel_for(T, [&](int64_t t) {
        for (int64_t c = 0; c < H; ++c) {
            double acc = y[(T * k + t) * H + c];
            for (int32_t j = 0; j < k; ++j) acc += w[t * k + j] * y[static_cast<int64_t>(perm_row[t * k + j]) * H + c];
            out[t * H + c] = acc;
        }
    });
    return 0;
}

// The timed CPU baseline: `repeats` passes of route + the sparse layer over x [T][H], timed with
// std::chrono::steady_clock; *seconds receives the elapsed wall time of all passes.
int so_forward_timed(const double* x, int64_t T, int64_t H, const double* w_router, int32_t E, const double* bias,
                     int32_t k, double scale, int64_t I, so_expert_fn fetch, void* ctx, double limit,
                     double limit_shared, int32_t repeats, double* out, double* seconds) {
    if (T <= 0 || repeats <= 0) return -1;
    const auto t0 = std::chrono::steady_clock::now();
    std::vector<double> L(T * E), s(T * E), bhat(T * E), w(T * k), gap(T);
    std::vector<int32_t> idx(T * k);
    for (int32_t rep = 0; rep < repeats; ++rep) {
        int rc = so_route(x, T, H, w_router, E, bias, k, scale, L.data(), s.data(), bhat.data(), idx.data(), w.data(),
                          gap.data());
        if (rc != 0) return rc;
        rc = so_moe(0, x, T, H, E, k, I, idx.data(), w.data(), fetch, ctx, limit, limit_shared, out);
        if (rc != 0) return rc;
    }
    *seconds = std::chrono::duration<double>(std::chrono::steady_clock::now() - t0).count();
    return 0;
}

}  // extern "C"
