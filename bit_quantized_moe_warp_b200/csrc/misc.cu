// misc.cu -- RMSNorm of the stack, the device-side packer of the 2-bit
// format, and the bounded-wait self test.
#include "common.cuh"
#include "kernels.h"

namespace strata {

// ------------------------------------------------------------ RMSNorm
// Stack glue (the layer recurrence x <- x + MoE(RMSNorm(x)) with unit
// weights): out = bf16_rne(x / sqrt(mean(x^2) + eps)), one block per token.
// sqrtf and the division are the IEEE-rounded operations.
__global__ void __launch_bounds__(256) k_rmsnorm_bf16(const float *__restrict__ x, __nv_bfloat16 *__restrict__ out,
                                                       int d, float eps) {
    __shared__ float red[8];
    const float *xr = x + (size_t)blockIdx.x * d;
    float ss = 0.f;
    for (int i = threadIdx.x; i < d; i += 256) ss = fmaf(xr[i], xr[i], ss);
    ss = warp_sum(ss);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x < 32) {
        float v = threadIdx.x < 8 ? red[threadIdx.x] : 0.f;
        v = warp_sum(v);
        if (threadIdx.x == 0) red[0] = v;
    }
    __syncthreads();
    const float inv = 1.0f / sqrtf(red[0] / (float)d + eps);
    for (int i = threadIdx.x; i < d; i += 256) out[(size_t)blockIdx.x * d + i] = __float2bfloat16_rn(xr[i] * inv);
}

void launch_rmsnorm_bf16(const float *x, void *out, int T, int d, float eps, cudaStream_t st) {
    if (T <= 0) return;
    k_rmsnorm_bf16<<<T, 256, 0, st>>>(x, static_cast<__nv_bfloat16 *>(out), d, eps);
}

// ------------------------------------------------------------ packer
// One thread per (tile, row): 64 codes -> the row's code words, then its two
// block scales. Column c = 16j + 8s + 2t + h: 2-bit, word t at bit
// 16h + 8s + 6 - 2j (four words); 4-bit, word 2t + j/2 at bit
// 16h + 8(j%2) + 4s (eight words). Tile (p, s) goes to
// dst + p * panel_stride + s * slice_stride.
template <int BITS>
__global__ void k_pack_matrix(const uint8_t *__restrict__ codes, const uint16_t *__restrict__ scales, int rows, int K,
                              uint8_t *__restrict__ dst, size_t panel_stride, size_t slice_stride) {
    using F = Qn<BITS>;
    const int slices = K / 64;
    const long long n = (long long)(rows / kTileRows) * slices * kTileRows;
    const long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= n) return;
    const int i = (int)(g % kTileRows);
    const long long tile = g / kTileRows;
    const int p = (int)(tile / slices), s = (int)(tile % slices);
    const int r = p * kTileRows + i;
    const uint8_t *cr = codes + (size_t)r * K + (size_t)s * 64;
    uint32_t w[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll 4
    for (int c = 0; c < 64; ++c) {
        const int j = c >> 4, sh = (c >> 3) & 1, tq = (c & 7) >> 1, h = c & 1;
        if (BITS == 4)
            w[2 * tq + (j >> 1)] |= (cr[c] & 15u) << (16 * h + 8 * (j & 1) + 4 * sh);
        else
            w[tq] |= (cr[c] & 3u) << (16 * h + 8 * sh + 6 - 2 * j);
    }
    uint8_t *t = dst + (size_t)p * panel_stride + (size_t)s * slice_stride;
    uint4 *tw = reinterpret_cast<uint4 *>(t + F::kRowBytes * i);
    tw[0] = make_uint4(w[0], w[1], w[2], w[3]);
    if (BITS == 4) tw[1] = make_uint4(w[4], w[5], w[6], w[7]);
    const uint16_t *sr = scales + (size_t)r * (K / 32) + 2 * s;
    *reinterpret_cast<uint32_t *>(t + F::kScaleOffset + 4 * i) = (uint32_t)sr[0] | ((uint32_t)sr[1] << 16);
}

void launch_pack_matrix_device(const uint8_t *codes, const uint16_t *scales, int rows, int K, int bits, uint8_t *dst,
                               size_t panel_stride, size_t slice_stride, cudaStream_t st) {
    const long long n = (long long)(rows / kTileRows) * (K / 64) * kTileRows;
    if (n <= 0) return;
    const unsigned grid = (unsigned)((n + 255) / 256);
    if (bits == 4)
        k_pack_matrix<4><<<grid, 256, 0, st>>>(codes, scales, rows, K, dst, panel_stride, slice_stride);
    else
        k_pack_matrix<2><<<grid, 256, 0, st>>>(codes, scales, rows, K, dst, panel_stride, slice_stride);
}

// ------------------------------------------------------------ self test
// Waits on a barrier that nothing arrives on; the bounded wait gives up
// after timeout_ns and records the timeout in the status word.
__global__ void k_wait_selftest(uint32_t *status, uint64_t timeout_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        mbar_wait(&bar, 0, status, nullptr, timeout_ns);
    }
}

void launch_wait_selftest(uint32_t *status, uint64_t timeout_ns, cudaStream_t st) {
    k_wait_selftest<<<1, 32, 0, st>>>(status, timeout_ns);
}

}  // namespace strata

namespace strata {

__global__ void k_bounds_selftest(uint32_t *status) {
    __shared__ int arr[16];
    const int idx = 16 + (int)threadIdx.x;  // one past the end
    arr[threadIdx.x & 15] = 1;
    if (in_bounds(idx, 16, status)) arr[idx & 15] += 1;  // never taken in the checked build
}

void launch_bounds_selftest(uint32_t *status, cudaStream_t st) { k_bounds_selftest<<<1, 1, 0, st>>>(status); }

}  // namespace strata
