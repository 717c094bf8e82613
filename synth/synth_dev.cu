// synth_dev.cu -- device twin of the seeded input generator in
// synth/__init__.py (same counter-based definition, bit-identical output).
// It only draws inputs; it holds none of the layer's arithmetic.
//
// word(key, i) = mix64(key + (i + 1) * GAMMA), mix64 = SplitMix64 output
// function. Codes: word i gives codes 32i..32i+31 (2-bit fields, LSB first),
// or 4-bit codes 16i..16i+15.
// Normal i: Irwin-Hall over the 12 20-bit fields of words 4i..4i+3, exact
// in float32; every later step is one IEEE round-to-nearest operation.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define GAMMA 0x9E3779B97F4A7C15ull

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

__device__ __forceinline__ uint64_t word(uint64_t key, uint64_t i) { return mix64(key + (i + 1) * GAMMA); }

__device__ __forceinline__ float normal(uint64_t key, uint64_t i) {
    int64_t s = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint64_t w = word(key, 4 * i + j);
        s += (int64_t)(w & 0xFFFFFull) + (int64_t)((w >> 20) & 0xFFFFFull) + (int64_t)((w >> 40) & 0xFFFFFull);
    }
    return __fmul_rn((float)(s - 6 * (1 << 20)), 9.5367431640625e-07f);  // * 2^-20, exact
}

// out[j * n + i] = code i of stream keys[j]; one thread per 32 codes (n % 32 == 0)
__global__ void k_codes(const uint64_t *keys, int64_t n, uint8_t *out) {
    const int j = blockIdx.y;
    const int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (w * 32 >= n) return;
    const uint64_t v = word(keys[j], (uint64_t)w);
    uint32_t b[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        uint32_t x = 0;
#pragma unroll
        for (int r = 0; r < 4; ++r) x |= (uint32_t)((v >> (2 * (4 * q + r))) & 3u) << (8 * r);
        b[q] = x;
    }
    uint4 *o = reinterpret_cast<uint4 *>(out + (size_t)j * n + (size_t)w * 32);
    o[0] = make_uint4(b[0], b[1], b[2], b[3]);
    o[1] = make_uint4(b[4], b[5], b[6], b[7]);
}

// 4-bit codes: one thread per 16 codes (n % 16 == 0), word i -> codes 16i..16i+15
__global__ void k_codes4(const uint64_t *keys, int64_t n, uint8_t *out) {
    const int j = blockIdx.y;
    const int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (w * 16 >= n) return;
    const uint64_t v = word(keys[j], (uint64_t)w);
    uint32_t b[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint32_t x = 0;
#pragma unroll
        for (int r = 0; r < 4; ++r) x |= (uint32_t)((v >> (4 * (4 * q + r))) & 15u) << (8 * r);
        b[q] = x;
    }
    *reinterpret_cast<uint4 *>(out + (size_t)j * n + (size_t)w * 16) = make_uint4(b[0], b[1], b[2], b[3]);
}

// scales fp16(|0.02 z| + 1e-3), divided by `div` (1 for 2-bit, 5 for 4-bit codes)
__global__ void k_scales(const uint64_t *keys, int64_t n, float div, uint16_t *out) {
    const int j = blockIdx.y;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const float z = normal(keys[j], (uint64_t)i);
    float t = __fadd_rn(fabsf(__fmul_rn(0.02f, z)), 1e-3f);
    if (div != 1.0f) t = __fdiv_rn(t, div);
    out[(size_t)j * n + i] = __half_as_ushort(__float2half_rn(t));
}

// x ~ N(0,1) rounded to bf16, elements start..start+n-1 of the stream
__global__ void k_x_bf16(uint64_t key, int64_t start, int64_t n, uint16_t *out) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    out[i] = __bfloat16_as_ushort(__float2bfloat16_rn(normal(key, (uint64_t)(start + i))));
}

// router weights 0.02 z in fp32
__global__ void k_router_w(uint64_t key, int64_t n, float *out) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    out[i] = __fmul_rn(0.02f, normal(key, (uint64_t)i));
}

extern "C" {

int synth_codes(const uint64_t *keys_dev, int nkeys, int64_t n, uint8_t *out, cudaStream_t st) {
    if (n % 32) return -1;
    dim3 grid((unsigned)((n / 32 + 255) / 256), nkeys);
    k_codes<<<grid, 256, 0, st>>>(keys_dev, n, out);
    return (int)cudaGetLastError();
}

int synth_codes4(const uint64_t *keys_dev, int nkeys, int64_t n, uint8_t *out, cudaStream_t st) {
    if (n % 16) return -1;
    dim3 grid((unsigned)((n / 16 + 255) / 256), nkeys);
    k_codes4<<<grid, 256, 0, st>>>(keys_dev, n, out);
    return (int)cudaGetLastError();
}

int synth_scales(const uint64_t *keys_dev, int nkeys, int64_t n, float div, uint16_t *out, cudaStream_t st) {
    dim3 grid((unsigned)((n + 255) / 256), nkeys);
    k_scales<<<grid, 256, 0, st>>>(keys_dev, n, div, out);
    return (int)cudaGetLastError();
}

int synth_x_bf16(uint64_t key, int64_t start, int64_t n, uint16_t *out, cudaStream_t st) {
    k_x_bf16<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(key, start, n, out);
    return (int)cudaGetLastError();
}

int synth_router_w(uint64_t key, int64_t n, float *out, cudaStream_t st) {
    k_router_w<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(key, n, out);
    return (int)cudaGetLastError();
}
}
