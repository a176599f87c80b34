/*
 * Seeded synthetic inputs, host side.
 *
 * This file holds none of the MoE layer's arithmetic. It produces the seeded
 * random tensors (activations, router weights, expert weights) that both the
 * CPU oracle and the CUDA library are fed, so the two sides see bit-identical
 * inputs. The device twin in synth_dev.cu implements the same definition.
 *
 * Definition (counter-based, so any slice can be produced independently):
 *   mix64(z)          = the splitmix64 finaliser (Vigna, "Further scramblings
 *                       of Marsaglia's xorshift generators"; shifts 30/27/31,
 *                       multipliers 0xBF58476D1CE4E5B9, 0x94D049BB133111EB)
 *   key(seed, tid)    = mix64(seed * G + tid),   G = 0x9E3779B97F4A7C15
 *   h_r(i)            = mix64(key + (2 i + r + 1) * G),   r = 0, 1
 *   S(i)              = sum of the eight 16-bit fields of h_0(i) and h_1(i)
 *   c(i)              = 2 S(i) - 8 * 65535          (an integer, |c| < 2^20)
 *   z(i)              = fp32(c(i)) * scale          (one fp32 multiply, RN)
 * c has mean 0 and standard deviation sqrt(8 * (65536^2 - 1) / 3); scale is
 * std / that value rounded to fp32 by the caller, so z is an Irwin-Hall(8)
 * approximation of N(0, std^2), bounded at about 4.9 std. bf16 tensors round
 * z to nearest-even. Every step is exact integer work or one IEEE fp32
 * multiply, so host and device agree bit for bit.
 *
 * Build: gcc -O3 -fopenmp -shared -fPIC synth_host.c -o libsmoe_synth_host.so
 */
#include <stdint.h>
#include <string.h>

#define SYNTH_G 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z ^= z >> 30;
    z *= 0xBF58476D1CE4E5B9ULL;
    z ^= z >> 27;
    z *= 0x94D049BB133111EBULL;
    z ^= z >> 31;
    return z;
}

static inline int32_t centred_sum(uint64_t key, uint64_t i) {
    uint64_t h0 = mix64(key + (2 * i + 1) * SYNTH_G);
    uint64_t h1 = mix64(key + (2 * i + 2) * SYNTH_G);
    int64_t s = 0;
    for (int f = 0; f < 4; ++f) {
        s += (int64_t)((h0 >> (16 * f)) & 0xFFFF);
        s += (int64_t)((h1 >> (16 * f)) & 0xFFFF);
    }
    return (int32_t)(2 * s - 8 * 65535);
}

static inline float as_float(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static inline uint32_t as_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u = as_bits(f);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

uint64_t synth_key(uint64_t seed, uint64_t tid) { return mix64(seed * SYNTH_G + tid); }

/* out[j] = z(index_base + j) as fp32, j in [0, n). scale_bits: fp32 bit pattern. */
void synth_host_fill_f32(float* out, int64_t n, uint64_t seed, uint64_t tid,
                         uint64_t index_base, uint32_t scale_bits) {
    const uint64_t key = synth_key(seed, tid);
    const float scale = as_float(scale_bits);
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j) {
        float c = (float)centred_sum(key, index_base + (uint64_t)j);
        out[j] = c * scale;
    }
}

/* out[j] = bf16_rne(z(index_base + j)) as raw bf16 bits. */
void synth_host_fill_bf16(uint16_t* out, int64_t n, uint64_t seed, uint64_t tid,
                          uint64_t index_base, uint32_t scale_bits) {
    const uint64_t key = synth_key(seed, tid);
    const float scale = as_float(scale_bits);
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j) {
        float c = (float)centred_sum(key, index_base + (uint64_t)j);
        float z = c * scale;
        out[j] = f32_to_bf16_rne(z);
    }
}

/* The raw 64-bit hash of counter i (used to rank rows/experts for seeded
 * sampling without replacement: take the rows with the smallest hashes). */
void synth_host_hash(uint64_t* out, int64_t n, uint64_t seed, uint64_t tid) {
    const uint64_t key = synth_key(seed, tid);
    for (int64_t j = 0; j < n; ++j) out[j] = mix64(key + (2 * (uint64_t)j + 1) * SYNTH_G);
}
