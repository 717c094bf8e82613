// decode.cu -- expert computation for 1..16 tokens (decode / draft verify).
//
// A decode step verifies 1 + up to 3 draft tokens in one pass ("Strata：把 125B
// 大模型塞进 12GB 显卡…", 投机解码); each token uses 10 experts (核心思路).
// At these sizes the layer is bound by the bytes of the selected experts'
// packed weights, so this path streams exactly those bytes once: 1-D bulk
// (TMA) copies of whole contiguous tile runs into shared memory, register
// dequantisation of the 2-bit codes, fp32 FMA against the tokens of the
// expert, and no tensor cores.
//
// Three kernels: gate/up partial sums per K split, SwiGLU + down projection
// per output panel and K split, and a deterministic per-token combine.
#include "common.cuh"
#include "kernels.h"

namespace strata {

// (c - 1.5) exactly, from a 2-bit code c: 2^22 + c is built by placing 2c in
// the mantissa of 2^22 (ulp 0.5), and 2^22 + 1.5 is subtracted.
STRATA_DEV float code_to_f(uint32_t c) { return __int_as_float(0x4A800000u | (c << 1)) - 4194305.5f; }

STRATA_DEV float2 scales2(uint32_t s) {
    __half2 h = *reinterpret_cast<__half2 *>(&s);
    return __half22float2(h);
}

// ------------------------------------------------------------ gate / up
// Work item = (active expert u, 128-row panel p of gate and up, K split ks).
// Thread (m, row) owns row `row` of matrix m (0 gate, 1 up) of the panel and
// accumulates its dot products with every token of the expert over the
// item's K range.
template <int TT>
__global__ void __launch_bounds__(256) k_decode_gateup(Workspace ws, const __nv_bfloat16 *__restrict__ x,
                                                        const uint8_t *__restrict__ blob, size_t ebytes, int T,
                                                        int d, int f, int KS, int NPD) {
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ uint64_t bar[2];
    __shared__ int s_abort;
    float *xs = reinterpret_cast<float *>(smem);
    const int SL = (d / 64) / KS;
    const uint32_t ibytes = (uint32_t)SL * 5120u;
    uint8_t *wbuf = smem + (((size_t)T * d * 4 + 1023) & ~(size_t)1023);
    const int P = f / 128;
    const int n_items = ws.meta[META_N_ACTIVE] * P * KS;
    const int tid = threadIdx.x;

    for (int i = tid; i < T * d; i += blockDim.x) xs[i] = __bfloat162float(x[i]);
    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        s_abort = 0;
        fence_mbar_init();
    }
    __syncthreads();

    uint32_t issued[2] = {0, 0}, waited[2] = {0, 0};  // thread 0's copy bookkeeping
    auto issue = [&](int item, int buf) {
        const int u = item / (P * KS), rem = item % (P * KS), p = rem / KS, ks = rem % KS;
        const int e = ws.act[u];
        const uint8_t *src = blob + (size_t)e * ebytes + ((size_t)p * (d / 64) + (size_t)ks * SL) * 5120;
        mbar_arrive_expect_tx(&bar[buf], ibytes);
        bulk_g2s(wbuf + (size_t)buf * ibytes, src, ibytes, &bar[buf]);
        ++issued[buf];
    };
    if (tid == 0 && (int)blockIdx.x < n_items) issue(blockIdx.x, 0);

    const int m = tid >> 7, row = tid & 127;
    int it = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++it) {
        const int buf = it & 1;
        if (tid == 0 && item + (int)gridDim.x < n_items) issue(item + gridDim.x, buf ^ 1);
        if (mbar_wait(&bar[buf], (it >> 1) & 1, ws.status, &s_abort) && tid == 0) ++waited[buf];
        __syncthreads();
        if (s_abort) break;

        const int u = item / (P * KS), rem = item % (P * KS), p = rem / KS, ks = rem % KS;
        const int e = ws.act[u];
        const int cnt = ws.counts[e], off = ws.offsets[e];
        int tok[TT];
#pragma unroll
        for (int i = 0; i < TT; ++i) tok[i] = (i < cnt) ? ws.token_list[off + i] : 0;
        float acc[TT];
#pragma unroll
        for (int i = 0; i < TT; ++i) acc[i] = 0.f;

        const uint8_t *tb = wbuf + (size_t)buf * ibytes + m * 2560;
        for (int sl = 0; sl < SL; ++sl) {
            const uint8_t *tile = tb + (size_t)sl * 5120;
            const uint4 cw = *reinterpret_cast<const uint4 *>(tile + 16 * row);
            const float2 sc = scales2(*reinterpret_cast<const uint32_t *>(tile + 2048 + 4 * row));
            const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
            const int col0 = (ks * SL + sl) * 64;
#pragma unroll
            for (int blk = 0; blk < 2; ++blk) {
                float bacc[TT];
#pragma unroll
                for (int i = 0; i < TT; ++i) bacc[i] = 0.f;
#pragma unroll
                for (int qq = 0; qq < 2; ++qq) {
                    const int q = 2 * blk + qq;
                    const uint32_t w = words[q];
#pragma unroll
                    for (int mp = 0; mp < 8; ++mp) {
                        const float fe = code_to_f((w >> (2 * mp)) & 3u);
                        const float fo = code_to_f((w >> (16 + 2 * mp)) & 3u);
                        const int col = col0 + 16 * q + 2 * mp;
#pragma unroll
                        for (int i = 0; i < TT; ++i) {
                            if (i < cnt) {
                                const float2 xv = *reinterpret_cast<const float2 *>(xs + (size_t)tok[i] * d + col);
                                bacc[i] = fmaf(fe, xv.x, bacc[i]);
                                bacc[i] = fmaf(fo, xv.y, bacc[i]);
                            }
                        }
                    }
                }
                const float s = blk ? sc.y : sc.x;
#pragma unroll
                for (int i = 0; i < TT; ++i) acc[i] = fmaf(s, bacc[i], acc[i]);
            }
        }
#pragma unroll
        for (int i = 0; i < TT; ++i)
            if (i < cnt) ws.gu_part[((size_t)(ks * NPD + off + i) * 2 + m) * f + p * 128 + row] = acc[i];
        __syncthreads();  // everyone is done with wbuf[buf] before it is refilled
    }
    if (tid == 0)  // after an abort: let copies still in flight land before exit
        for (int b = 0; b < 2; ++b)
            while (waited[b] < issued[b]) {
                mbar_wait(&bar[b], waited[b] & 1, ws.status, nullptr);
                ++waited[b];
            }
}

// ------------------------------------------------------------ down
// Work item = (active expert u, 128-row panel p of down, K split kd). The
// block first forms h = silu(g) * u for the expert's tokens on its K range
// (summing the gate/up partials), then thread `row` computes the panel row's
// dot products with h for every token.
template <int TT>
__global__ void __launch_bounds__(128) k_decode_down(Workspace ws, const uint8_t *__restrict__ blob, size_t ebytes,
                                                      size_t down_off, int T, int d, int f, int KS, int NPD) {
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ uint64_t bar[2];
    __shared__ int s_abort;
    const int FH = f / kDecKSD;  // K range of one split
    const int SLD = FH / 64;
    const uint32_t ibytes = (uint32_t)SLD * 2560u;
    uint8_t *wbuf = smem;
    float *hs = reinterpret_cast<float *>(smem + 2 * (size_t)ibytes);  // [TT][FH]
    const int P = d / 128;
    const int n_items = ws.meta[META_N_ACTIVE] * P * kDecKSD;
    const int tid = threadIdx.x;
    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        s_abort = 0;
        fence_mbar_init();
    }
    __syncthreads();
    uint32_t issued[2] = {0, 0}, waited[2] = {0, 0};  // thread 0's copy bookkeeping
    auto issue = [&](int item, int buf) {
        const int u = item / (P * kDecKSD), rem = item % (P * kDecKSD), p = rem / kDecKSD, kd = rem % kDecKSD;
        const int e = ws.act[u];
        const uint8_t *src =
            blob + (size_t)e * ebytes + down_off + ((size_t)p * (f / 64) + (size_t)kd * SLD) * 2560;
        mbar_arrive_expect_tx(&bar[buf], ibytes);
        bulk_g2s(wbuf + (size_t)buf * ibytes, src, ibytes, &bar[buf]);
        ++issued[buf];
    };
    if (tid == 0 && (int)blockIdx.x < n_items) issue(blockIdx.x, 0);

    int it = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++it) {
        const int buf = it & 1;
        if (tid == 0 && item + (int)gridDim.x < n_items) issue(item + gridDim.x, buf ^ 1);
        const int u = item / (P * kDecKSD), rem = item % (P * kDecKSD), p = rem / kDecKSD, kd = rem % kDecKSD;
        const int e = ws.act[u];
        const int cnt = ws.counts[e], off = ws.offsets[e];
        for (int idx = tid; idx < cnt * FH; idx += blockDim.x) {
            const int i = idx / FH, r = idx % FH;
            const int col = kd * FH + r;
            float g = 0.f, uu = 0.f;
            for (int ks = 0; ks < KS; ++ks) {
                const size_t base = (size_t)(ks * NPD + off + i) * 2 * f + col;
                g += ws.gu_part[base];
                uu += ws.gu_part[base + f];
            }
            hs[i * FH + r] = silu_f(g) * uu;
        }
        if (mbar_wait(&bar[buf], (it >> 1) & 1, ws.status, &s_abort) && tid == 0) ++waited[buf];
        __syncthreads();
        if (s_abort) break;
        float acc[TT];
#pragma unroll
        for (int i = 0; i < TT; ++i) acc[i] = 0.f;
        const int row = tid;
        for (int sl = 0; sl < SLD; ++sl) {
            const uint8_t *tile = wbuf + (size_t)buf * ibytes + (size_t)sl * 2560;
            const uint4 cw = *reinterpret_cast<const uint4 *>(tile + 16 * row);
            const float2 sc = scales2(*reinterpret_cast<const uint32_t *>(tile + 2048 + 4 * row));
            const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
            for (int blk = 0; blk < 2; ++blk) {
                float bacc[TT];
#pragma unroll
                for (int i = 0; i < TT; ++i) bacc[i] = 0.f;
#pragma unroll
                for (int qq = 0; qq < 2; ++qq) {
                    const int q = 2 * blk + qq;
                    const uint32_t w = words[q];
#pragma unroll
                    for (int mp = 0; mp < 8; ++mp) {
                        const float fe = code_to_f((w >> (2 * mp)) & 3u);
                        const float fo = code_to_f((w >> (16 + 2 * mp)) & 3u);
                        const int col = sl * 64 + 16 * q + 2 * mp;
#pragma unroll
                        for (int i = 0; i < TT; ++i) {
                            if (i < cnt) {
                                const float2 hv = *reinterpret_cast<const float2 *>(hs + i * FH + col);
                                bacc[i] = fmaf(fe, hv.x, bacc[i]);
                                bacc[i] = fmaf(fo, hv.y, bacc[i]);
                            }
                        }
                    }
                }
                const float s = blk ? sc.y : sc.x;
#pragma unroll
                for (int i = 0; i < TT; ++i) acc[i] = fmaf(s, bacc[i], acc[i]);
            }
        }
#pragma unroll
        for (int i = 0; i < TT; ++i)
            if (i < cnt) ws.o_part[(size_t)(kd * NPD + off + i) * d + p * 128 + row] = acc[i];
        __syncthreads();
    }
    if (tid == 0)
        for (int b = 0; b < 2; ++b)
            while (waited[b] < issued[b]) {
                mbar_wait(&bar[b], waited[b] & 1, ws.status, nullptr);
                ++waited[b];
            }
}

// ------------------------------------------------------------ combine
// y[t] (=|+=) sum_j w[t][j] * sum_kd o_part[kd][pair(t, j)], in slot order.
__global__ void __launch_bounds__(256) k_decode_combine(Workspace ws, float *__restrict__ y, int d, int k, int NPD,
                                                         int accumulate) {
    const int t = blockIdx.y;
    const int c = blockIdx.x * 256 + threadIdx.x;
    if (c >= d) return;
    float v = accumulate ? y[(size_t)t * d + c] : 0.f;
    for (int j = 0; j < k; ++j) {
        const int p = ws.pair_of[t * k + j];
        const float w = ws.topk_w[t * k + j];
        float o = 0.f;
        for (int kd = 0; kd < kDecKSD; ++kd) o += ws.o_part[(size_t)(kd * NPD + p) * d + c];
        v = fmaf(w, o, v);
    }
    y[(size_t)t * d + c] = v;
}

template <int TT>
static void decode_impl(const Workspace &ws, const void *x, const uint8_t *blob, float *y, bool accumulate, int T,
                        const Shape &s, int num_sms, cudaStream_t st, cudaEvent_t *ev) {
    const size_t eb = expert_bytes(s);
    const int KS = ((s.d / 64) % kDecKS == 0) ? kDecKS : 2;
    const int NPD = kDecMaxT * s.k;
    const int SL = (s.d / 64) / KS;
    const size_t smem1 = (((size_t)T * s.d * 4 + 1023) & ~(size_t)1023) + 2 * (size_t)SL * 5120;
    if (ev) cudaEventRecord(ev[2], st);
    k_decode_gateup<TT><<<num_sms, 256, smem1, st>>>(ws, static_cast<const __nv_bfloat16 *>(x), blob, eb, T, s.d,
                                                     s.f, KS, NPD);
    if (ev) cudaEventRecord(ev[3], st);
    const int FH = s.f / kDecKSD, SLD = FH / 64;
    const size_t smem2 = 2 * (size_t)SLD * 2560 + (size_t)TT * FH * 4;
    k_decode_down<TT><<<num_sms * 2, 128, smem2, st>>>(ws, blob, eb, down_section_offset(s), T, s.d, s.f, KS, NPD);
    dim3 g3((s.d + 255) / 256, T);
    k_decode_combine<<<g3, 256, 0, st>>>(ws, y, s.d, s.k, NPD, accumulate ? 1 : 0);
}

void init_decode_attributes(int max_smem) {
    cudaFuncSetAttribute(k_decode_gateup<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
    cudaFuncSetAttribute(k_decode_gateup<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
    cudaFuncSetAttribute(k_decode_gateup<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
    cudaFuncSetAttribute(k_decode_down<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
    cudaFuncSetAttribute(k_decode_down<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
    cudaFuncSetAttribute(k_decode_down<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
}

void launch_decode_experts(const Workspace &ws, const void *x, const uint8_t *blob, float *y, bool accumulate,
                           int T, const Shape &s, int num_sms, cudaStream_t st, cudaEvent_t *ev) {
    if (T <= 1)
        decode_impl<1>(ws, x, blob, y, accumulate, T, s, num_sms, st, ev);
    else if (T <= 4)
        decode_impl<4>(ws, x, blob, y, accumulate, T, s, num_sms, st, ev);
    else
        decode_impl<16>(ws, x, blob, y, accumulate, T, s, num_sms, st, ev);
}

}  // namespace strata
