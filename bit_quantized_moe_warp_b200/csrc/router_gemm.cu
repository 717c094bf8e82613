// router_gemm.cu -- router logits for prefill sizes on the 5th-generation
// tensor cores: logits[T x E] = x W_r^T (+ bias).
//
// The router ("Strata：把 125B 大模型塞进 12GB 显卡…", 代码结构: a router kernel
// on the GPU) takes fp32 weights and bf16 activations. The tensor cores
// multiply bf16 operands exactly into fp32, so W_r is split once per call
// into two bf16 parts, W = hi + lo + r with |r| <= 2^-18 |W| (hi the bf16
// rounding of W, lo the bf16 rounding of W - hi), and both parts multiply x
// (bf16, exact) into one fp32 accumulator: the logits carry at most
// 2^-18 sum_i |x_i W_i| of representation error plus fp32 accumulation.
//
// Tiles of 128 experts x 256 tokens, K in 64-column steps: warp 0 issues
// 2-D tensor copies (128-byte swizzle) of W_hi, W_lo and x; warp 1 issues
// tcgen05.mma kind::f16 (bf16 inputs, fp32 accumulators in tensor memory,
// double-buffered); warps 2-5 read the accumulators, add the bias and store
// the logits. Every wait is time-bounded and unwinds through the status word.
#include "common.cuh"
#include "kernels.h"

namespace strata {

constexpr int kRgM = 128, kRgN = 256, kRgStages = 3, kRgThreads = 192;
constexpr uint32_t kRgA = kRgM * 64 * 2;  // one bf16 W tile (128 rows x 64 columns)
constexpr uint32_t kRgB = kRgN * 64 * 2;  // one bf16 x tile (256 rows x 64 columns)
constexpr uint32_t kRgStage = 2 * kRgA + kRgB;
constexpr uint32_t kRgSmem = kRgStages * kRgStage + 1024;  // + alignment slack
constexpr uint32_t kRgTmemCols = 2 * kRgN;

// instruction descriptor: fp32 accumulator, bf16 A and B, both K-major
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__global__ void __launch_bounds__(kRgThreads, 1)
    k_router_tc(const __grid_constant__ CUtensorMap mw_hi, const __grid_constant__ CUtensorMap mw_lo,
                const __grid_constant__ CUtensorMap mx, const float *__restrict__ bias, float *__restrict__ logits,
                int T, int E, int d, uint32_t *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full[kRgStages], empty[kRgStages], accfull[2], accempty[2], fin;
    __shared__ uint32_t tmem_base;
    __shared__ int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int mt = (E + kRgM - 1) / kRgM, nt = (T + kRgN - 1) / kRgN;
    const int n_items = mt * nt, KSTEPS = d / 64;
    auto A_at = [&](int st, int part) { return smem + (size_t)st * kRgStage + (size_t)part * kRgA; };
    auto B_at = [&](int st) { return smem + (size_t)st * kRgStage + 2 * kRgA; };

    if (threadIdx.x == 0) {
        for (int i = 0; i < kRgStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&accfull[i], 1);
            mbar_init(&accempty[i], 4);
        }
        mbar_init(&fin, 1);
        s_abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&mw_hi);
        prefetch_tmap(&mw_lo);
        prefetch_tmap(&mx);
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base, kRgTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = tmem_base;

    if (warp == 0) {
        // ------------------------------------------------ tensor copies
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
                const int m0 = (item % mt) * kRgM, n0 = (item / mt) * kRgN;
                for (int ks = 0; ks < KSTEPS; ++ks, ++it) {
                    const int st = it % kRgStages;
                    if (!mbar_wait(&empty[st], ((it / kRgStages) & 1) ^ 1, status, &s_abort)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[st], kRgStage);
                    tma_load_2d(A_at(st, 0), &mw_hi, ks * 64, m0, &full[st]);
                    tma_load_2d(A_at(st, 1), &mw_lo, ks * 64, m0, &full[st]);
                    tma_load_2d(B_at(st), &mx, ks * 64, n0, &full[st]);
                }
            }
            // copies still in flight (only after an abort) land before exit
            const uint32_t first = it > (uint32_t)kRgStages ? it - kRgStages : 0;
            for (uint32_t j = first; j < it; ++j) mbar_wait(&full[j % kRgStages], (j / kRgStages) & 1, status, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issue
        if (lane == 0) {
            const uint32_t idesc = umma_idesc_bf16(kRgM, kRgN);
            uint32_t it = 0, li = 0;
            bool ok = true;
            for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x, ++li) {
                const int acc = li & 1;
                if (!mbar_wait(&accempty[acc], ((li >> 1) & 1) ^ 1, status, &s_abort)) break;
                tc_fence_after();
                const uint32_t dcol = tbase + (uint32_t)(acc * kRgN);
                for (int ks = 0; ks < KSTEPS; ++ks, ++it) {
                    const int st = it % kRgStages;
                    if (!mbar_wait(&full[st], (it / kRgStages) & 1, status, &s_abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ahi = umma_desc_sw128(A_at(st, 0)), alo = umma_desc_sw128(A_at(st, 1));
                    const uint64_t bd = umma_desc_sw128(B_at(st));
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        umma_f16(dcol, ahi + 2 * kk, bd + 2 * kk, idesc, (ks | kk) ? 1u : 0u);
                        umma_f16(dcol, alo + 2 * kk, bd + 2 * kk, idesc, 1u);
                    }
                    umma_commit(&empty[st]);
                }
                if (ok) umma_commit(&accfull[acc]);
            }
            umma_commit(&fin);  // every MMA of this thread is complete before tensor memory is freed
            mbar_wait(&fin, 0, status, nullptr);
        }
    } else {
        // ------------------------------------------------ epilogue: bias, store
        const int q = warp & 3;  // tensor-memory lanes 32q .. 32q + 31
        uint32_t li = 0;
        for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++li) {
            const int m0 = (item % mt) * kRgM, n0 = (item / mt) * kRgN;
            const int acc = li & 1;
            if (!mbar_wait(&accfull[acc], (li >> 1) & 1, status, &s_abort)) break;
            tc_fence_after();
            const int e = m0 + 32 * q + lane;
            const float b = (bias && e < E) ? bias[e] : 0.f;
            const uint32_t trow = tbase + ((uint32_t)(32 * q) << 16) + (uint32_t)(acc * kRgN);
            for (int c0 = 0; c0 < kRgN; c0 += 16) {
                if (n0 + c0 >= T) break;
                float v[16];
                tmem_ld16(trow + c0, v);
                tmem_ld_wait();
                if (e < E) {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (n0 + c0 + i < T) logits[(size_t)(n0 + c0 + i) * E + e] = v[i] + b;
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&accempty[acc]);
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, kRgTmemCols);
    }
}

// W (fp32) -> hi = bf16(W), lo = bf16(W - hi)
__global__ void __launch_bounds__(256) k_split_router(const float4 *__restrict__ W, uint2 *__restrict__ hi,
                                                      uint2 *__restrict__ lo, size_t n4) {
    for (size_t i = (size_t)blockIdx.x * 256 + threadIdx.x; i < n4; i += (size_t)gridDim.x * 256) {
        const float4 w = W[i];
        const float v[4] = {w.x, w.y, w.z, w.w};
        __nv_bfloat16 h[4], l[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            h[j] = __float2bfloat16_rn(v[j]);
            l[j] = __float2bfloat16_rn(v[j] - __bfloat162float(h[j]));
        }
        hi[i] = *reinterpret_cast<const uint2 *>(h);
        lo[i] = *reinterpret_cast<const uint2 *>(l);
    }
}

cudaError_t init_router_attributes(int max_smem) {
    if ((int)kRgSmem > max_smem) return cudaErrorInvalidValue;
    return cudaFuncSetAttribute(k_router_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRgSmem);
}

void launch_router_tc(const Workspace &ws, const RouterMaps &maps, const float *W, const float *bias, float *logits,
                      int T, const Shape &s, int num_sms, cudaStream_t st) {
    const size_t n4 = (size_t)s.E * s.d / 4;
    k_split_router<<<(unsigned)((n4 + 255) / 256 < 1184 ? (n4 + 255) / 256 : 1184), 256, 0, st>>>(
        reinterpret_cast<const float4 *>(W), static_cast<uint2 *>(ws.w_hi), static_cast<uint2 *>(ws.w_lo), n4);
    const int items = ((s.E + kRgM - 1) / kRgM) * ((T + kRgN - 1) / kRgN);
    const int grid = items < num_sms ? items : num_sms;
    k_router_tc<<<grid, kRgThreads, kRgSmem, st>>>(maps.w_hi, maps.w_lo, maps.x, bias, logits, T, s.E, s.d,
                                                    ws.status);
}

}  // namespace strata
