// kv_codec.cu -- the 4-bit Hadamard-rotated KV-cache codec of include/strata_kv.h
// ("Strata：把 125B 大模型塞进 12GB 显卡…", sections 长上下文 and 代码结构).
//
// Both kernels stream rows from HBM once and write each result once; they are
// bound by HBM bandwidth (encode: 2 + 0.5625 bytes per value, decode the
// reverse), with the transform's butterflies and the block rule in registers.
//
// Value layout in a warp: a row of D values is spread over D / (8 R)
// consecutive lanes (R = 4 runs of 8 values per lane for D >= 128, 2 for
// D = 64): lane l (of its row) holds values 8 (l + m D / (8 R)) + e for runs
// m < R and e < 8. One 16-byte load per run: a warp instruction reads
// D / (8 R) x 16 contiguous bytes of each of its rows. Index bits 0..2 (e)
// and the top log2(R) bits (m) are inside the lane; the bits in between (l)
// are crossed with one shuffle per value and stage (2, 2, 3 stages for
// D = 64, 128, 256). The butterfly stages run in the order of their stride,
// 1, 2, ..., D/2, each pair (a, b) becoming (a + b, a - b) in fp32, which
// fixes every rounding of the encoder; from stride 2 on, two butterflies go
// through one packed fp32x2 instruction. A 32-value quantisation block is 4
// lanes x 8 values: its absmax takes two xor-shuffles.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/strata_kv.h"
#include "abi_internal.h"

namespace {

constexpr int kThreads = 256;
constexpr unsigned kFull = 0xffffffffu;
// 1.5 * 2^23 + 8: added to p with |p| < 2^22 it leaves rint(p) + 8 (ties to
// even) in the low mantissa bits
constexpr float kRound8 = 12582920.f;

template <int D>
struct KvRow {
    static constexpr int kRuns = D == 64 ? 2 : 4;        // runs of 8 values per lane
    static constexpr int kLanes = D / (8 * kRuns);       // lanes per row
    static constexpr int kRowsPerWarp = 32 / kLanes;     // rows per warp instruction
    static constexpr int kUnroll = 4 / kRuns;            // row groups in flight per warp
    static constexpr int kVec = D / 8;                   // 16-byte chunks of bf16 (and 4-byte code words) per row
    static constexpr int kBlocks = D / 32;               // scales per row
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

__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }

// (a + b, a - b) on two butterflies at once; a - b = fma(-1, b, a) exactly
__device__ __forceinline__ void bfly2(float2 &a, float2 &b) {
    const float2 s = __fadd2_rn(a, b);
    b = __ffma2_rn(f2(-1.f), b, a);
    a = s;
}

// Unnormalised Walsh-Hadamard transform of the row whose values this lane
// holds, x[m][k] = (value 2k, value 2k + 1) of run m; lane l of the row.
template <int D>
__device__ __forceinline__ void fwht_row(float2 (&x)[KvRow<D>::kRuns][4], int l) {
    using R = KvRow<D>;
#pragma unroll
    for (int m = 0; m < R::kRuns; ++m)
#pragma unroll
        for (int k = 0; k < 4; ++k) {  // stride 1: the two halves of a pair
            const float a = x[m][k].x, b = x[m][k].y;
            x[m][k] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
        }
#pragma unroll
    for (int m = 0; m < R::kRuns; ++m) {
        bfly2(x[m][0], x[m][1]);  // stride 2
        bfly2(x[m][2], x[m][3]);
        bfly2(x[m][0], x[m][2]);  // stride 4
        bfly2(x[m][1], x[m][3]);
    }
#pragma unroll
    for (int k = 1; k < R::kLanes; k <<= 1) {
        // the lane with bit k of l clear holds a, its partner b: the lower lane
        // forms a + b, the upper p - v = a - b (the sign flip is exact)
        const float2 sg = f2((l & k) ? -1.f : 1.f);
#pragma unroll
        for (int m = 0; m < R::kRuns; ++m)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 p = make_float2(__shfl_xor_sync(kFull, x[m][j].x, k), __shfl_xor_sync(kFull, x[m][j].y, k));
                x[m][j] = __ffma2_rn(sg, x[m][j], p);
            }
    }
#pragma unroll
    for (int h = 1; h < R::kRuns; h <<= 1)  // the run bits, lowest first
#pragma unroll
        for (int m = 0; m < R::kRuns; ++m)
            if (!(m & h))
#pragma unroll
                for (int j = 0; j < 4; ++j) bfly2(x[m][j], x[m + h][j]);
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 w, float2 (&v)[4]) {
    const uint32_t p[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = make_float2(__uint_as_float(p[k] << 16), __uint_as_float(p[k] & 0xffff0000u));
}

// Codes of one run from the rounded sums z (low nibbles): byte j of the word
// holds value 2j in its low nibble and 2j + 1 in its high one.
__device__ __forceinline__ uint32_t pack_nibbles(const uint32_t (&z)[8]) {
    const uint32_t even = __byte_perm(__byte_perm(z[0], z[2], 0x0040), __byte_perm(z[4], z[6], 0x4000), 0x7610);
    const uint32_t odd = __byte_perm(__byte_perm(z[1], z[3], 0x0040), __byte_perm(z[5], z[7], 0x4000), 0x7610);
    return even | (odd << 4);
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
    for (int64_t g0 = warp * R::kUnroll; g0 < n_groups; g0 += n_warps * R::kUnroll) {  // warp-uniform
        uint4 raw[R::kUnroll][R::kRuns];
#pragma unroll
        for (int u = 0; u < R::kUnroll; ++u) {
            const int64_t row = (g0 + u) * R::kRowsPerWarp + rw;
#pragma unroll
            for (int m = 0; m < R::kRuns; ++m)
                raw[u][m] = row < n_rows ? __ldcs(x + row * R::kVec + l + R::kLanes * m) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < R::kUnroll; ++u) {
            const int64_t row = (g0 + u) * R::kRowsPerWarp + rw;
            float2 v[R::kRuns][4];
#pragma unroll
            for (int m = 0; m < R::kRuns; ++m) bf16x8_to_f32(raw[u][m], v[m]);
            fwht_row<D>(v, l);
            uint32_t word[R::kRuns];
            uint16_t sbits[R::kRuns];
            float amax[R::kRuns];
#pragma unroll
            for (int m = 0; m < R::kRuns; ++m) {
                amax[m] = 0.f;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    v[m][k] = __fmul2_rn(v[m][k], f2(r));
                    amax[m] = fmaxf(amax[m], fmaxf(fabsf(v[m][k].x), fabsf(v[m][k].y)));
                }
                amax[m] = fmaxf(amax[m], __shfl_xor_sync(kFull, amax[m], 1));
                amax[m] = fmaxf(amax[m], __shfl_xor_sync(kFull, amax[m], 2));
            }
            // Block scales. With 4 runs a warp holds 8 blocks x 4 runs = 32 (block,
            // run) pairs, and every lane of a block already has the block's absmax
            // for each run: lane j computes the scale of run j % 4 of its block once,
            // and the block's lanes fetch the four results (instead of each lane
            // computing all four, four times per block).
            float inv_of[R::kRuns];
            uint32_t sw_of[R::kRuns];  // scale bits | 1 << 16 when the scale is a normal half
            {
                float a = amax[0];
#pragma unroll
                for (int m = 1; m < R::kRuns; ++m) a = (lane % R::kRuns) == m ? amax[m] : a;
                float inv = 0.f;
                uint32_t sw = 0;
                if (R::kRuns == 4) {
                    const float t = __fdiv_rn(a, 7.f);
                    const __half hs = __float2half_rn(fminf(t, 65504.f));
                    const float sv = __half2float(hs);
                    inv = sv > 0.f ? __frcp_rn(sv) : 0.f;
                    sw = __half_as_ushort(hs) | ((t >= 6.103515625e-05f && t <= 65504.f) ? 0x10000u : 0u);
                }
#pragma unroll
                for (int m = 0; m < R::kRuns; ++m) {
                    if (R::kRuns == 4) {
                        inv_of[m] = __shfl_sync(kFull, inv, (lane & ~3) + m);
                        sw_of[m] = __shfl_sync(kFull, sw, (lane & ~3) + m);
                    } else {  // two runs: each lane computes its own
                        const float t = __fdiv_rn(amax[m], 7.f);
                        const __half hs = __float2half_rn(fminf(t, 65504.f));
                        const float sv = __half2float(hs);
                        inv_of[m] = sv > 0.f ? __frcp_rn(sv) : 0.f;
                        sw_of[m] = __half_as_ushort(hs) | ((t >= 6.103515625e-05f && t <= 65504.f) ? 0x10000u : 0u);
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < R::kRuns; ++m) {
                const float inv = inv_of[m];
                uint32_t z[8];
                if (sw_of[m] >> 16) {
                    // s is a normal half within 2^-11 of absmax / 7: |y * inv| < 7.5,
                    // so one fused multiply-add rounds the exact product, no clamp
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float2 q = __ffma2_rn(v[m][k], f2(inv), f2(kRound8));
                        z[2 * k] = __float_as_uint(q.x);
                        z[2 * k + 1] = __float_as_uint(q.y);
                    }
                } else {
                    // a subnormal or saturated scale: the product may leave [-7.5, 7.5]
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float y = (e & 1) ? v[m][e / 2].y : v[m][e / 2].x;
                        int q;
                        if (fabsf(__fmul_rn(y, inv)) >= 8.f) {
                            q = y > 0.f ? 7 : -7;  // the exact product is beyond 7.5
                        } else {
                            q = (int)(__float_as_uint(__fmaf_rn(y, inv, 12582912.f)) - 0x4b400000u);
                            q = q > 7 ? 7 : (q < -7 ? -7 : q);
                        }
                        z[e] = (uint32_t)(q + 8);
                    }
                }
                word[m] = pack_nibbles(z);
                sbits[m] = (uint16_t)sw_of[m];
            }
            if (row < n_rows) {
#pragma unroll
                for (int m = 0; m < R::kRuns; ++m) {
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
    for (int64_t g0 = warp * R::kUnroll; g0 < n_groups; g0 += n_warps * R::kUnroll) {  // warp-uniform
        uint32_t w[R::kUnroll][R::kRuns];
        uint16_t sb[R::kUnroll][R::kRuns];
#pragma unroll
        for (int u = 0; u < R::kUnroll; ++u) {
            const int64_t row = (g0 + u) * R::kRowsPerWarp + rw;
#pragma unroll
            for (int m = 0; m < R::kRuns; ++m) {
                const bool ok = row < n_rows;
                w[u][m] = ok ? __ldcs(codes + row * R::kVec + l + R::kLanes * m) : 0x88888888u;
                sb[u][m] = ok ? __ldcs(scales + row * R::kBlocks + (l + R::kLanes * m) / 4) : (uint16_t)0;
            }
        }
#pragma unroll
        for (int u = 0; u < R::kUnroll; ++u) {
            const int64_t row = (g0 + u) * R::kRowsPerWarp + rw;
            float2 v[R::kRuns][4];
#pragma unroll
            for (int m = 0; m < R::kRuns; ++m) {
                // (c - 8) * s * fp32(1/sqrt(D)): the normalisation is applied on the
                // way in (the transform is linear)
                const float sr = __fmul_rn(__half2float(__ushort_as_half(sb[u][m])), r);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    // 2^23 + c, minus 2^23 + 8: the exact c - 8
                    const float2 c = make_float2(__uint_as_float(0x4b000000u | ((w[u][m] >> (8 * k)) & 15u)),
                                                 __uint_as_float(0x4b000000u | ((w[u][m] >> (8 * k + 4)) & 15u)));
                    v[m][k] = __fmul2_rn(__fadd2_rn(c, f2(-8388616.f)), f2(sr));
                }
            }
            fwht_row<D>(v, l);
            if (row < n_rows) {
#pragma unroll
                for (int m = 0; m < R::kRuns; ++m) {
                    uint32_t o[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[m][k].x, v[m][k].y);
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
int grid_for(K kernel, int64_t n_rows, int rows_per_warp, int unroll, int device) {
    int sms = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || sms <= 0) sms = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, 0) != cudaSuccess || per_sm <= 0)
        per_sm = 1;
    const int64_t groups = (n_rows + rows_per_warp - 1) / rows_per_warp;
    const int64_t warps = (groups + unroll - 1) / unroll;
    const int64_t need = (warps + kThreads / 32 - 1) / (kThreads / 32);
    const int64_t cap = (int64_t)sms * per_sm;
    return (int)(need < cap ? need : cap);
}

template <int D>
cudaError_t launch_encode(const void *x, int64_t n, void *codes, void *scales, cudaStream_t st) {
    int dev = 0;
    cudaGetDevice(&dev);
    const int grid = grid_for(k_kv4_encode<D>, n, KvRow<D>::kRowsPerWarp, KvRow<D>::kUnroll, dev);
    k_kv4_encode<D><<<grid, kThreads, 0, st>>>(static_cast<const uint4 *>(x), n, static_cast<uint32_t *>(codes),
                                              static_cast<uint16_t *>(scales));
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_decode(const void *codes, const void *scales, int64_t n, void *out, cudaStream_t st) {
    int dev = 0;
    cudaGetDevice(&dev);
    const int grid = grid_for(k_kv4_decode<D>, n, KvRow<D>::kRowsPerWarp, KvRow<D>::kUnroll, dev);
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
