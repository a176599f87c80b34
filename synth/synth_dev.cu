// Seeded synthetic inputs, device side: the twin of synth_host.c.
//
// This file holds none of the MoE layer's arithmetic. It writes the same
// counter-based Irwin-Hall(8) values as synth_host.c straight into device
// memory, so multi-GB expert weights never cross PCIe. The definition is
// stated in synth_host.c; every step here is integer work or one fp32
// multiply written with __fmul_rn, so both sides agree bit for bit.
//
// Build: nvcc -gencode arch=compute_100a,code=sm_100a -O3 -shared
//        -Xcompiler -fPIC synth_dev.cu -o libsmoe_synth_dev.so
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#define SYNTH_G 0x9E3779B97F4A7C15ULL

__host__ __device__ static inline uint64_t mix64(uint64_t z) {
    z ^= z >> 30;
    z *= 0xBF58476D1CE4E5B9ULL;
    z ^= z >> 27;
    z *= 0x94D049BB133111EBULL;
    z ^= z >> 31;
    return z;
}

__device__ static inline int32_t centred_sum(uint64_t key, uint64_t i) {
    uint64_t h0 = mix64(key + (2 * i + 1) * SYNTH_G);
    uint64_t h1 = mix64(key + (2 * i + 2) * SYNTH_G);
    int64_t s = 0;
#pragma unroll
    for (int f = 0; f < 4; ++f) {
        s += (int64_t)((h0 >> (16 * f)) & 0xFFFF);
        s += (int64_t)((h1 >> (16 * f)) & 0xFFFF);
    }
    return (int32_t)(2 * s - 8 * 65535);
}

__device__ static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u = __float_as_uint(f);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

__global__ void synth_fill_f32_kernel(float* out, int64_t n, uint64_t key, uint64_t base, float scale) {
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < n;
         j += (int64_t)gridDim.x * blockDim.x) {
        float c = (float)centred_sum(key, base + (uint64_t)j);
        out[j] = __fmul_rn(c, scale);
    }
}

__global__ void synth_fill_bf16_kernel(uint16_t* out, int64_t n, uint64_t key, uint64_t base, float scale) {
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < n;
         j += (int64_t)gridDim.x * blockDim.x) {
        float c = (float)centred_sum(key, base + (uint64_t)j);
        out[j] = f32_to_bf16_rne(__fmul_rn(c, scale));
    }
}

static int grid_for(int64_t n) {
    int64_t blocks = (n + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    return (int)blocks;
}

extern "C" {

// Returns 0 on success, else the cudaError_t of the launch.
int synth_dev_fill_f32(float* out, int64_t n, uint64_t seed, uint64_t tid, uint64_t index_base,
                       uint32_t scale_bits, cudaStream_t stream) {
    if (n <= 0) return 0;
    float scale;
    memcpy(&scale, &scale_bits, 4);
    uint64_t key = mix64(seed * SYNTH_G + tid);
    synth_fill_f32_kernel<<<grid_for(n), 256, 0, stream>>>(out, n, key, index_base, scale);
    return (int)cudaGetLastError();
}

int synth_dev_fill_bf16(uint16_t* out, int64_t n, uint64_t seed, uint64_t tid, uint64_t index_base,
                        uint32_t scale_bits, cudaStream_t stream) {
    if (n <= 0) return 0;
    float scale;
    memcpy(&scale, &scale_bits, 4);
    uint64_t key = mix64(seed * SYNTH_G + tid);
    synth_fill_bf16_kernel<<<grid_for(n), 256, 0, stream>>>(out, n, key, index_base, scale);
    return (int)cudaGetLastError();
}

}  // extern "C"
