// kv_codec.cu -- the 4-bit Hadamard-rotated KV-cache codec of include/strata_kv.h
// ("Strata：把 125B 大模型塞进 12GB 显卡…", sections 长上下文 and 代码结构).
//
// Both kernels stream rows from HBM once and write each result once; they are
// bound by HBM bandwidth (encode: 2 + 0.5625 bytes per value, decode the
// reverse), with the transform's butterflies and the block rule in registers.
//
// Value layout in a warp: a row of D values is spread over D/16 consecutive
// lanes, each holding 16 values as two runs of 8: lane l (of its row) holds
// values 8 (l + m D/16) + e, m in {0, 1}, e in [0, 8). One 16-byte load per
// run: a warp instruction reads D/16 x 16 contiguous bytes of each of its
// rows. Index bits 0..2 (e) and the top bit (m) are inside the lane; the
// bits in between (l) are crossed with one shuffle per value and stage, so a
// row needs log2(D/16) shuffle stages (2, 3, 4 for D = 64, 128, 256). The
// butterfly stages run in the order of their stride, 1, 2, ..., D/2, each
// pair (a, b) becoming (a + b, a - b) in fp32, which fixes every rounding of
// the encoder. A 32-value quantisation block is 4 lanes x 8 values: its
// absmax takes two xor-shuffles.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/strata_kv.h"
#include "abi_internal.h"

namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 2;  // row groups whose loads a warp issues before computing
constexpr unsigned kFull = 0xffffffffu;

template <int D>
struct KvRow {
    static constexpr int kLanes = D / 16;              // lanes per row
    static constexpr int kRowsPerWarp = 32 / kLanes;   // rows per warp instruction
    static constexpr int kVec = D / 8;                 // 16-byte chunks of bf16 (and 4-byte code words) per row
    static constexpr int kBlocks = D / 32;             // scales per row
};

// fp32(1 / sqrt(D)), the rotation's normalisation
template <int D>
__device__ __forceinline__ float inv_sqrt_d();
template <>
__device__ __forceinline__ float inv_sqrt_d<64>() { return 0.125f; }
template <>
__device__ __forceinline__ float inv_sqrt_d<128>() { return 0.08838834764831844055f; }
template <>
__device__ __forceinline__ float inv_sqrt_d<256>() { return 0.0625f; }

// Unnormalised Walsh-Hadamard transform of the row whose values v[m][e] this
// lane holds (lane l of the row), stage strides 1, 2, ..., D/2 in order.
template <int D>
__device__ __forceinline__ void fwht_row(float (&v)[2][8], int l) {
#pragma unroll
    for (int h = 1; h < 8; h <<= 1)
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int e = 0; e < 8; ++e)
                if (!(e & h)) {
                    const float a = v[m][e], b = v[m][e + h];
                    v[m][e] = __fadd_rn(a, b);
                    v[m][e + h] = __fsub_rn(a, b);
                }
#pragma unroll
    for (int k = 1; k < KvRow<D>::kLanes; k <<= 1) {
        // the lane with bit k of l clear holds a, its partner b: the lower lane
        // forms a + b, the upper p - v = a - b (the sign flip is exact)
        const float sg = (l & k) ? -1.f : 1.f;
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float p = __shfl_xor_sync(kFull, v[m][e], k);
                v[m][e] = __fmaf_rn(sg, v[m][e], p);
            }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const float a = v[0][e], b = v[1][e];
        v[0][e] = __fadd_rn(a, b);
        v[1][e] = __fsub_rn(a, b);
    }
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 w, float (&v)[8]) {
    const uint32_t p[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        v[2 * k] = __uint_as_float(p[k] << 16);
        v[2 * k + 1] = __uint_as_float(p[k] & 0xffff0000u);
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads) k_kv4_encode(const uint4 *__restrict__ x, int64_t n_rows,
                                                        uint32_t *__restrict__ codes, uint16_t *__restrict__ scales) {
    using R = KvRow<D>;
    const int lane = threadIdx.x & 31, l = lane % R::kLanes, rw = lane / R::kLanes;
    const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * kThreads) >> 5;
    const int64_t n_groups = (n_rows + R::kRowsPerWarp - 1) / R::kRowsPerWarp;
    const float r = inv_sqrt_d<D>();
    for (int64_t g0 = warp * kUnroll; g0 < n_groups; g0 += n_warps * kUnroll) {  // warp-uniform
        uint4 raw[kUnroll][2];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t row = (g0 + u) * R::kRowsPerWarp + rw;
#pragma unroll
            for (int m = 0; m < 2; ++m)
                raw[u][m] = row < n_rows ? __ldcs(x + row * R::kVec + l + R::kLanes * m) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t row = (g0 + u) * R::kRowsPerWarp + rw;
            float v[2][8];
            bf16x8_to_f32(raw[u][0], v[0]);
            bf16x8_to_f32(raw[u][1], v[1]);
            fwht_row<D>(v, l);
            uint32_t word[2];
            uint16_t sbits[2];
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                float amax = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    v[m][e] = __fmul_rn(v[m][e], r);
                    amax = fmaxf(amax, fabsf(v[m][e]));
                }
                amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
                amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
                const __half hs = __float2half_rn(fminf(__fdiv_rn(amax, 7.f), 65504.f));
                const float s = __half2float(hs);
                const float inv = s > 0.f ? __frcp_rn(s) : 0.f;
                uint32_t wd = 0;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    // clamp, then round half to even by adding 1.5 * 2^23 + 8:
                    // the sum's low mantissa bits are rint(p) + 8 in [1, 15]
                    const float p = fminf(fmaxf(__fmul_rn(v[m][e], inv), -7.f), 7.f);
                    wd |= (__float_as_uint(__fadd_rn(p, 12582920.f)) & 15u) << (4 * e);
                }
                word[m] = wd;
                sbits[m] = __half_as_ushort(hs);
            }
            if (row < n_rows) {
#pragma unroll
                for (int m = 0; m < 2; ++m) {
                    __stcs(codes + row * R::kVec + l + R::kLanes * m, word[m]);
                    if ((l & 3) == 0) __stcs(scales + row * R::kBlocks + (l + R::kLanes * m) / 4, sbits[m]);
                }
            }
        }
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads) k_kv4_decode(const uint32_t *__restrict__ codes,
                                                        const uint16_t *__restrict__ scales, int64_t n_rows,
                                                        uint4 *__restrict__ out) {
    using R = KvRow<D>;
    const int lane = threadIdx.x & 31, l = lane % R::kLanes, rw = lane / R::kLanes;
    const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * kThreads) >> 5;
    const int64_t n_groups = (n_rows + R::kRowsPerWarp - 1) / R::kRowsPerWarp;
    const float r = inv_sqrt_d<D>();
    for (int64_t g0 = warp * kUnroll; g0 < n_groups; g0 += n_warps * kUnroll) {  // warp-uniform
        uint32_t w[kUnroll][2];
        uint16_t sb[kUnroll][2];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t row = (g0 + u) * R::kRowsPerWarp + rw;
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const bool ok = row < n_rows;
                w[u][m] = ok ? __ldcs(codes + row * R::kVec + l + R::kLanes * m) : 0x88888888u;
                sb[u][m] = ok ? __ldcs(scales + row * R::kBlocks + (l + R::kLanes * m) / 4) : (uint16_t)0;
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t row = (g0 + u) * R::kRowsPerWarp + rw;
            float v[2][8];
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const float s = __half2float(__ushort_as_half(sb[u][m]));
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    // 2^23 + c, minus 2^23 + 8: the exact c - 8
                    const float q = __fsub_rn(__uint_as_float(0x4b000000u | ((w[u][m] >> (4 * e)) & 15u)), 8388616.f);
                    v[m][e] = __fmul_rn(q, s);
                }
            }
            fwht_row<D>(v, l);
            if (row < n_rows) {
#pragma unroll
                for (int m = 0; m < 2; ++m) {
                    uint32_t o[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const __nv_bfloat162 b2 =
                            __floats2bfloat162_rn(__fmul_rn(v[m][2 * k], r), __fmul_rn(v[m][2 * k + 1], r));
                        o[k] = *reinterpret_cast<const uint32_t *>(&b2);
                    }
                    __stcs(out + row * R::kVec + l + R::kLanes * m, make_uint4(o[0], o[1], o[2], o[3]));
                }
            }
        }
    }
}

// Blocks for n_rows rows: enough warps for every row group, at most the
// number the device holds at once (a persistent grid-stride loop beyond that).
template <typename K>
int grid_for(K kernel, int64_t n_rows, int rows_per_warp, int device) {
    int sms = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || sms <= 0) sms = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, 0) != cudaSuccess || per_sm <= 0)
        per_sm = 1;
    const int64_t groups = (n_rows + rows_per_warp - 1) / rows_per_warp;
    const int64_t warps = (groups + kUnroll - 1) / kUnroll;
    const int64_t need = (warps + kThreads / 32 - 1) / (kThreads / 32);
    const int64_t cap = (int64_t)sms * per_sm;
    return (int)(need < cap ? need : cap);
}

template <int D>
cudaError_t launch_encode(const void *x, int64_t n, void *codes, void *scales, cudaStream_t st) {
    int dev = 0;
    cudaGetDevice(&dev);
    const int grid = grid_for(k_kv4_encode<D>, n, KvRow<D>::kRowsPerWarp, dev);
    k_kv4_encode<D><<<grid, kThreads, 0, st>>>(static_cast<const uint4 *>(x), n, static_cast<uint32_t *>(codes),
                                              static_cast<uint16_t *>(scales));
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_decode(const void *codes, const void *scales, int64_t n, void *out, cudaStream_t st) {
    int dev = 0;
    cudaGetDevice(&dev);
    const int grid = grid_for(k_kv4_decode<D>, n, KvRow<D>::kRowsPerWarp, dev);
    k_kv4_decode<D><<<grid, kThreads, 0, st>>>(static_cast<const uint32_t *>(codes),
                                              static_cast<const uint16_t *>(scales), n, static_cast<uint4 *>(out));
    return cudaGetLastError();
}

bool supported_dim(int32_t D) { return D == 64 || D == 128 || D == 256; }

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" size_t strata_kv4_code_bytes(int64_t n_rows, int32_t head_dim) {
    return (n_rows > 0 && supported_dim(head_dim)) ? (size_t)n_rows * (size_t)(head_dim / 2) : 0;
}

extern "C" size_t strata_kv4_scale_bytes(int64_t n_rows, int32_t head_dim) {
    return (n_rows > 0 && supported_dim(head_dim)) ? (size_t)n_rows * (size_t)(head_dim / 32) * 2 : 0;
}

extern "C" strata_status strata_kv4_encode(const void *x, int64_t n_rows, int32_t head_dim, void *codes,
                                           void *scales, strata_stream_t stream) {
    if (!supported_dim(head_dim)) return strata_set_error(STRATA_ERR_UNSUPPORTED, "head_dim %d not in {64, 128, 256}", head_dim);
    if (n_rows < 0) return strata_set_error(STRATA_ERR_INVALID_ARG, "n_rows %lld < 0", (long long)n_rows);
    if (n_rows == 0) return STRATA_OK;
    if (!x || !codes || !scales) return strata_set_error(STRATA_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned(x, 16) || !aligned(codes, 4) || !aligned(scales, 2))
        return strata_set_error(STRATA_ERR_INVALID_ARG, "x must be 16-byte, codes 4-byte, scales 2-byte aligned");
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = head_dim == 64    ? launch_encode<64>(x, n_rows, codes, scales, st)
                    : head_dim == 128 ? launch_encode<128>(x, n_rows, codes, scales, st)
                                      : launch_encode<256>(x, n_rows, codes, scales, st);
    if (e != cudaSuccess) return strata_set_error(STRATA_ERR_CUDA, "kv4 encode launch: %s", cudaGetErrorString(e));
    return STRATA_OK;
}

extern "C" strata_status strata_kv4_decode(const void *codes, const void *scales, int64_t n_rows, int32_t head_dim,
                                           void *out, strata_stream_t stream) {
    if (!supported_dim(head_dim)) return strata_set_error(STRATA_ERR_UNSUPPORTED, "head_dim %d not in {64, 128, 256}", head_dim);
    if (n_rows < 0) return strata_set_error(STRATA_ERR_INVALID_ARG, "n_rows %lld < 0", (long long)n_rows);
    if (n_rows == 0) return STRATA_OK;
    if (!codes || !scales || !out) return strata_set_error(STRATA_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned(out, 16) || !aligned(codes, 4) || !aligned(scales, 2))
        return strata_set_error(STRATA_ERR_INVALID_ARG, "out must be 16-byte, codes 4-byte, scales 2-byte aligned");
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = head_dim == 64    ? launch_decode<64>(codes, scales, n_rows, out, st)
                    : head_dim == 128 ? launch_decode<128>(codes, scales, n_rows, out, st)
                                      : launch_decode<256>(codes, scales, n_rows, out, st);
    if (e != cudaSuccess) return strata_set_error(STRATA_ERR_CUDA, "kv4 decode launch: %s", cudaGetErrorString(e));
    return STRATA_OK;
}
