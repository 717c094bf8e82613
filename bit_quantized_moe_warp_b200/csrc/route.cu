// route.cu -- router logits, softmax top-k and per-expert token lists.
//
// Router ("Strata：把 125B 大模型塞进 12GB 显卡…", 代码结构: a router kernel on
// the GPU; 10 experts per token, 核心思路). The layer's specification fixes
// the rest: logits = W_r x (+ bias), softmax over the layer's experts, the k
// largest with ties to the lower expert index, probabilities renormalised
// over the k selected, and per-expert token lists for the expert kernels.
#include "common.cuh"
#include "kernels.h"
#include "topk.cuh"

namespace strata {

// ------------------------------------------------------------ router GEMV
// Decode sizes (T <= 16): one warp per expert row, 16-byte coalesced loads
// of W_r, fp32 FMA, a fixed per-row reduction order (identical rows give
// bit-identical logits, which the tie rule relies on).
template <int TT>
__global__ void __launch_bounds__(128) k_router_gemv(const __nv_bfloat16 *__restrict__ x,
                                                      const float *__restrict__ W,
                                                      const float *__restrict__ bias, float *__restrict__ logits,
                                                      int T, int d, int E) {
    const int lane = threadIdx.x & 31;
    const int e = blockIdx.x * 4 + (threadIdx.x >> 5);
    if (e >= E) return;
    float acc[TT];
#pragma unroll
    for (int t = 0; t < TT; ++t) acc[t] = 0.f;
    const float4 *w4 = reinterpret_cast<const float4 *>(W + (size_t)e * d);
    for (int i = lane; i < d / 4; i += 32) {
        float4 w = __ldg(w4 + i);
#pragma unroll
        for (int t = 0; t < TT; ++t) {
            if (t < T) {
                const uint2 xr = *reinterpret_cast<const uint2 *>(x + (size_t)t * d + 4 * i);
                float x0 = __uint_as_float(xr.x << 16), x1 = __uint_as_float(xr.x & 0xffff0000u);
                float x2 = __uint_as_float(xr.y << 16), x3 = __uint_as_float(xr.y & 0xffff0000u);
                acc[t] = fmaf(w.x, x0, acc[t]);
                acc[t] = fmaf(w.y, x1, acc[t]);
                acc[t] = fmaf(w.z, x2, acc[t]);
                acc[t] = fmaf(w.w, x3, acc[t]);
            }
        }
    }
    const float b = bias ? bias[e] : 0.f;
#pragma unroll
    for (int t = 0; t < TT; ++t) {
        float v = warp_sum(acc[t]);
        if (lane == 0 && t < T) logits[(size_t)t * E + e] = v + b;
    }
}

// ------------------------------------------------------------ top-k
// One warp per token: lane l owns experts l, l+32, ... (E <= 1024). k rounds
// of a warp arg-max over (logit descending, index ascending); only the
// winning lane rescans its own values. Then w_j = exp(l_j - l_max) /
// sum_{j'} exp(l_j' - l_max), which equals the softmax over all experts
// renormalised over the selected ones.
__device__ __forceinline__ bool rank_better(float v, int i, float bv, int bi) {
    return v > bv || (v == bv && i < bi);
}

__device__ void warp_topk(const float *__restrict__ lrow, int E, int k, int *sel_idx, float *sel_w) {
    const int lane = threadIdx.x & 31;
    float v[32];
    uint32_t taken = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = (lane + 32 * i < E) ? lrow[lane + 32 * i] : 0.f;
    const int nmine = (E - lane + 31) / 32;  // values this lane owns
    auto local_best = [&](float &bv, int &bi) {
        bv = 0.f;
        bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if (i < nmine && !((taken >> i) & 1u)) {
                int idx = lane + 32 * i;
                if (bi == 0x7fffffff || rank_better(v[i], idx, bv, bi)) {
                    bv = v[i];
                    bi = idx;
                }
            }
        }
    };
    float bv;
    int bi;
    local_best(bv, bi);
    float myval = 0.f;
    int myidx = 0;
    float vmax = 0.f;
    for (int j = 0; j < k; ++j) {
        float wv = bv;
        int wi = bi;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            float ov = __shfl_xor_sync(0xffffffffu, wv, o);
            int oi = __shfl_xor_sync(0xffffffffu, wi, o);
            bool take = (oi != 0x7fffffff) && (wi == 0x7fffffff || rank_better(ov, oi, wv, wi));
            if (take) {
                wv = ov;
                wi = oi;
            }
        }
        if (j == 0) vmax = wv;
        if (lane == j) {
            myval = wv;
            myidx = wi;
        }
        if ((wi & 31) == lane) {
            taken |= 1u << (wi >> 5);
            local_best(bv, bi);
        }
    }
    float ex = (lane < k) ? expf(myval - vmax) : 0.f;
    float den = warp_sum(ex);
    if (lane < k) {
        sel_idx[lane] = myidx;
        sel_w[lane] = ex / den;
    }
}

// ------------------------------------------------------------ large lists
// Prefill sizes. (1) top-k per token, one warp per token; expert counts per
// 256-token block accumulated with atomics (blk_counts zeroed beforehand).
constexpr int kTopkTokensPerCta = 8;  // one token per warp
// With xs (the bf16 tokens) it also records each token's power-of-two scale
// for the fp16 expert operands in ws.tok_s.
__global__ void __launch_bounds__(256) k_topk_blocks(Workspace ws, const uint4 *__restrict__ xs, int d, int T, int E,
                                                     int k) {
    __shared__ int s_idx[8][32];
    __shared__ float s_w[8][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (blockIdx.x == 0 && threadIdx.x == 0) ws.meta[META_N_TOKENS] = T;
    const int t0 = blockIdx.x * kTopkTokensPerCta;
    for (int i = warp; i < kTopkTokensPerCta; i += 8) {
        const int t = t0 + i;
        if (t >= T) break;
        if (xs) {  // the token's largest |x| (from the bf16 bits) -> its scale
            uint32_t am = 0u;
            for (int c = lane; c < d / 8; c += 32) {
                const uint4 v = __ldg(xs + (size_t)t * (d / 8) + c);
                const uint32_t in[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) am = max(am, max(in[j] & 0x7fffu, (in[j] >> 16) & 0x7fffu));
            }
            am = __reduce_max_sync(0xffffffffu, am);
            if (lane == 0) ws.tok_s[t] = pow2_scale(__uint_as_float(am << 16));
        }
        if (E <= 512 && E % 4 == 0) {  // sorted per-lane lists, one warp max + ballot per pick
            token_topk<16>(ws.logits, t, E, k, s_idx[warp], s_w[warp]);
            __syncwarp();
            const float vmax = s_w[warp][0];
            const float ex = lane < k ? expf(s_w[warp][lane] - vmax) : 0.f;
            const float den = warp_sum(ex);
            __syncwarp();
            if (lane < k) s_w[warp][lane] = ex / den;
        } else {
            warp_topk(ws.logits + (size_t)t * E, E, k, s_idx[warp], s_w[warp]);
        }
        __syncwarp();
        if (lane < k) {
            const int e = s_idx[warp][lane];
            ws.topk_idx[(size_t)t * k + lane] = e;
            ws.topk_w[(size_t)t * k + lane] = s_w[warp][lane];
            if (in_bounds(e, E, ws.status)) atomicAdd(&ws.blk_counts[(size_t)(t / kRouteBlock) * E + e], 1);
        }
        __syncwarp();
    }
}

// (2) one block: expert totals, offsets, per-block bases (in place in
// blk_counts), and the GEMM tile lists: full tiles of all experts first,
// then the partial ones (largest work first).
__global__ void __launch_bounds__(1024) k_lists_scan(Workspace ws, int T, int E, int max_tiles1, int max_tiles2) {
    __shared__ int s_off[1025];
    __shared__ int s_f1[1025], s_p1[1025], s_f2[1025], s_p2[1025];
    const int nblk = (T + kRouteBlock - 1) / kRouteBlock;
    const int e = threadIdx.x;
    int tot = 0;
    if (e < E) {
        for (int b = 0; b < nblk; ++b) {
            int c = ws.blk_counts[(size_t)b * E + e];
            ws.blk_counts[(size_t)b * E + e] = tot;  // exclusive prefix over blocks
            tot += c;
        }
    }
    // exclusive scans over the experts of: the pair count, the full and the
    // partial gate/up tiles, the full and the partial down tiles (a block
    // scan: warp shuffles, then the warp totals)
    __shared__ int s_wsum[32][5];
    {
        const int t = e < E ? tot : 0;
        int v[5] = {t, t / kGemm1N, (t % kGemm1N) != 0, t / kGemm2N, (t % kGemm2N) != 0};
        int incl[5];
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
        for (int q = 0; q < 5; ++q) incl[q] = v[q];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1)
#pragma unroll
            for (int q = 0; q < 5; ++q) {
                const int u = __shfl_up_sync(0xffffffffu, incl[q], o);
                if (lane >= o) incl[q] += u;
            }
        if (lane == 31)
#pragma unroll
            for (int q = 0; q < 5; ++q) s_wsum[warp][q] = incl[q];
        __syncthreads();
        if (warp == 0) {
#pragma unroll
            for (int q = 0; q < 5; ++q) {
                int w = s_wsum[lane][q];  // 32 warps of 32 threads cover 1024 experts
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int u = __shfl_up_sync(0xffffffffu, w, o);
                    if (lane >= o) w += u;
                }
                s_wsum[lane][q] = w;  // inclusive over warps
            }
        }
        __syncthreads();
        int ex[5];
#pragma unroll
        for (int q = 0; q < 5; ++q) ex[q] = (warp ? s_wsum[warp - 1][q] : 0) + incl[q] - v[q];
        if (e < E) {
            s_off[e] = ex[0];
            s_f1[e] = ex[1];
            s_p1[e] = ex[2];
            s_f2[e] = ex[3];
            s_p2[e] = ex[4];
        }
        if (threadIdx.x == 0) {
            s_off[E] = s_wsum[31][0];
            s_f1[E] = s_wsum[31][1];
            s_p1[E] = s_wsum[31][2];
            s_f2[E] = s_wsum[31][3];
            s_p2[E] = s_wsum[31][4];
            ws.meta[META_N_TILES1] = min(s_wsum[31][1] + s_wsum[31][2], max_tiles1);
            ws.meta[META_N_TILES2] = min(s_wsum[31][3] + s_wsum[31][4], max_tiles2);
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) ws.offsets[E] = s_off[E];
    if (e < E) {
        ws.offsets[e] = s_off[e];
        ws.counts[e] = tot;
        for (int b = 0; b < nblk; ++b) ws.blk_counts[(size_t)b * E + e] += s_off[e];
        const int F1 = s_f1[E], F2 = s_f2[E];
        int nf = tot / kGemm1N;
        for (int i = 0; i < nf; ++i)
            if (s_f1[e] + i < max_tiles1)
                ws.tiles1[s_f1[e] + i] = make_int4(e, s_off[e] + i * kGemm1N, kGemm1N, 0);
        if (tot % kGemm1N && F1 + s_p1[e] < max_tiles1)
            ws.tiles1[F1 + s_p1[e]] = make_int4(e, s_off[e] + nf * kGemm1N, tot % kGemm1N, 0);
        nf = tot / kGemm2N;
        for (int i = 0; i < nf; ++i)
            if (s_f2[e] + i < max_tiles2)
                ws.tiles2[s_f2[e] + i] = make_int4(e, s_off[e] + i * kGemm2N, kGemm2N, 0);
        if (tot % kGemm2N && F2 + s_p2[e] < max_tiles2)
            ws.tiles2[F2 + s_p2[e]] = make_int4(e, s_off[e] + nf * kGemm2N, tot % kGemm2N, 0);
    }
}

// (3) stable scatter: within a 256-token block, a bitmap per expert of the
// tokens that chose it; the rank of (t, e) is the block base plus the number
// of earlier tokens of the block in e's bitmap.
__global__ void __launch_bounds__(256) k_lists_scatter(Workspace ws, int T, int E, int k) {
    extern __shared__ uint32_t s_bits[];  // [E][8]
    for (int i = threadIdx.x; i < E * 8; i += 256) s_bits[i] = 0u;
    __syncthreads();
    const int i = threadIdx.x;
    const int t = blockIdx.x * kRouteBlock + i;
    if (t < T)
        for (int j = 0; j < k; ++j) {
            int e = ws.topk_idx[(size_t)t * k + j];
            if (in_bounds(e, E, ws.status)) atomicOr(&s_bits[e * 8 + (i >> 5)], 1u << (i & 31));
        }
    __syncthreads();
    if (t < T)
        for (int j = 0; j < k; ++j) {
            int e = ws.topk_idx[(size_t)t * k + j];
            if (!in_bounds(e, E, ws.status)) continue;
            int r = __popc(s_bits[e * 8 + (i >> 5)] & ((1u << (i & 31)) - 1u));
            for (int w = 0; w < (i >> 5); ++w) r += __popc(s_bits[e * 8 + w]);
            int pos = ws.blk_counts[(size_t)blockIdx.x * E + e] + r;
            if (!in_bounds(pos, (long long)T * k, ws.status)) continue;
            ws.token_list[pos] = t;
            ws.pair_slot[pos] = j;
            ws.pair_w[pos] = ws.topk_w[(size_t)t * k + j];
            ws.pair_of[(size_t)t * k + j] = pos;
        }
}

// ------------------------------------------------------------ gather
// xp[p] = fp16(x[t] * s_t) for the pair's token t, with s_t the token's
// power-of-two scale (tok_s, from the routing), copied to pair_s[p]: one warp
// per pair row, 16-byte accesses.
__global__ void __launch_bounds__(256) k_gather_xp(const __nv_bfloat16 *__restrict__ x,
                                                    const int *__restrict__ token_list, const float *__restrict__ tok_s,
                                                    __half *__restrict__ xp, float *__restrict__ pair_s, int npairs,
                                                    int d, int T, uint32_t *status) {
    const int p = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (p >= npairs) return;
    const int t = token_list[p];
    if (!in_bounds(t, T, status)) return;
    const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)t * d);
    uint4 *dst = reinterpret_cast<uint4 *>(xp + (size_t)p * d);
    const float sc = tok_s[t];
    if (lane == 0) pair_s[p] = sc;
    for (int c = lane; c < d / 8; c += 32) {
        const uint4 v = __ldg(src + c);
        const uint32_t in[4] = {v.x, v.y, v.z, v.w};
        uint32_t out[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float lo = __uint_as_float(in[q] << 16) * sc, hi = __uint_as_float(in[q] & 0xffff0000u) * sc;
            __half2 h = __floats2half2_rn(lo, hi);
            out[q] = *reinterpret_cast<uint32_t *>(&h);
        }
        dst[c] = make_uint4(out[0], out[1], out[2], out[3]);
    }
}

// ------------------------------------------------------------ launchers
void launch_router_gemv(const void *x, const float *W, const float *bias, float *logits, int T, const Shape &s,
                        cudaStream_t st) {
    dim3 grid((s.E + 3) / 4), block(128);
    auto xb = static_cast<const __nv_bfloat16 *>(x);
    if (T <= 1)
        k_router_gemv<1><<<grid, block, 0, st>>>(xb, W, bias, logits, T, s.d, s.E);
    else if (T <= 4)
        k_router_gemv<4><<<grid, block, 0, st>>>(xb, W, bias, logits, T, s.d, s.E);
    else
        k_router_gemv<16><<<grid, block, 0, st>>>(xb, W, bias, logits, T, s.d, s.E);
}

void launch_route_large(const Workspace &ws, int T, int max_tiles1, int max_tiles2, const Shape &s,
                        cudaStream_t st, const void *x_scale_src) {
    const int nblk = (T + kRouteBlock - 1) / kRouteBlock;
    cudaMemsetAsync(ws.blk_counts, 0, (size_t)nblk * s.E * sizeof(int32_t), st);
    const uint4 *xs = ws.tok_s ? static_cast<const uint4 *>(x_scale_src) : nullptr;
    k_topk_blocks<<<(T + kTopkTokensPerCta - 1) / kTopkTokensPerCta, 256, 0, st>>>(ws, xs, s.d, T, s.E, s.k);
    k_lists_scan<<<1, 1024, 0, st>>>(ws, T, s.E, max_tiles1, max_tiles2);
    k_lists_scatter<<<nblk, 256, (size_t)s.E * 8 * sizeof(uint32_t), st>>>(ws, T, s.E, s.k);
}

void launch_gather_xp(const Workspace &ws, const void *x, int T, const Shape &s, cudaStream_t st) {
    const int np = T * s.k;
    k_gather_xp<<<(np + 7) / 8, 256, 0, st>>>(static_cast<const __nv_bfloat16 *>(x), ws.token_list, ws.tok_s,
                                               static_cast<__half *>(ws.xp), ws.pair_s, np, s.d, T, ws.status);
}

}  // namespace strata
