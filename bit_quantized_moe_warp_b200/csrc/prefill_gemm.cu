// prefill_gemm.cu -- grouped expert GEMMs on the 5th-generation tensor cores
// (tcgen05, accumulators in tensor memory) for prefill chunks, on 2-bit or
// 4-bit tiles.
//
// Prompts are read in chunks of up to 8,192 tokens and the expert products
// run on the quantised weights instead of first expanding them to FP16 in
// memory ("Strata：把 125B 大模型塞进 12GB 显卡…", 工程细节). Here every
// 128-row x 64-column block of 2-bit weights (two 64-row tiles) is copied once
// per token tile into shared memory (1-D bulk copies), dequantised there to fp16, and fed to
// tcgen05.mma; the tokens of one expert (a contiguous run of the gathered,
// expert-sorted rows) come in by 2-D tensor copies with 128-byte swizzle.
//
//   MODE 0 (gate/up + SwiGLU): per tile of <= 128 tokens and 128-row panel
//     of gate and up, two accumulators G, U [128 x N] share the token
//     operand; the epilogue writes H = silu(G) * U (fp16, pair-major).
//   MODE 1 (down): per tile of <= 256 pairs and 128-row panel of down,
//     O = W_down H^T; the epilogue stores O (fp16, pair-major) and a
//     combine kernel sums each token's k rows, weighted, into y (no atomics).
//
// Warp roles (448 threads): warp 0 issues the copies, warp 1 issues the MMAs
// (one thread), warps 2-5 drain the accumulators, warps 6-13 dequantise.
// Stage ring: full (copies landed) -> aready (dequant done) -> MMA ->
// empty (commit). Accumulators are double-buffered (accfull / accempty), so
// the epilogue of one tile overlaps the main loop of the next.
#include "common.cuh"
#include "kernels.h"

namespace strata {

// Stages: four, except gate/up on 4-bit tiles, whose four stages (57 KB
// each) would not fit in 227 KB of shared memory.
template <int MODE, int BITS>
struct GCfg;
template <int BITS>
struct GCfg<0, BITS> {
    static constexpr int NMAT = 2, NMAX = kGemm1N, STAGES = BITS == 4 ? 3 : 4;
};
template <int BITS>
struct GCfg<1, BITS> {
    static constexpr int NMAT = 1, NMAX = kGemm2N, STAGES = 4;
};

constexpr int kGemmThreads = 448;
constexpr int kDequantWarps = 8;

template <int MODE, int BITS>
struct GLayout {
    static constexpr int NMAT = GCfg<MODE, BITS>::NMAT, NMAX = GCfg<MODE, BITS>::NMAX,
                         STAGES = GCfg<MODE, BITS>::STAGES;
    static constexpr uint32_t TILE = Qn<BITS>::kTileBytes;
    static constexpr uint32_t A_BYTES = 128 * 64 * 2;  // one fp16 matrix tile
    static constexpr uint32_t B_BYTES = NMAX * 128;    // NMAX rows of 64 fp16
    static constexpr uint32_t W_BYTES = NMAT * 2 * TILE;  // packed tiles: 128 rows per matrix
    static constexpr uint32_t STAGE = ((NMAT * A_BYTES + B_BYTES + W_BYTES) + 1023) / 1024 * 1024;
    static constexpr uint32_t SMEM = STAGES * STAGE + 1024;  // + alignment slack
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(2 * NMAT * NMAX <= 512, "accumulators exceed tensor memory");
};

struct GemmArgs {
    const uint8_t *blob;
    size_t ebytes;     // bytes per expert
    size_t sec_off;    // byte offset of this GEMM's section inside an expert
    size_t tile_panel; // byte stride between 64-row tile panels of the section
    size_t tile_slice; // byte stride between 64-column K slices of the section
    int K;             // reduction length (d for MODE 0, f for MODE 1)
    int panels;        // 128-row panels of the output (f/128 or d/128)
    int ldo;           // MODE 0: f (row length of H); MODE 1: d (row length of y)
    const int4 *tiles;
    const int *n_tiles;
    __half *H;         // MODE 0 output
    __half *O;         // MODE 1 output: W_down h per pair [pairs x d]
    const float *pair_s;  // MODE 0: power-of-two scale of each pair's token (carried by the gathered x)
    int n_experts, n_pairs;   // bounds of the tile entries (checked build)
    uint32_t *status;
};

// A tile entry {expert, first pair, pairs, 0}; in the checked build a bad
// one is recorded and replaced by a harmless tile (expert 0, pairs from 0),
// the same way in every warp role so the pipelines stay in step.
template <int NMAX>
STRATA_DEV int4 tile_at(const GemmArgs &a, int i) {
    int4 tl = a.tiles[i];
    const bool ok = in_bounds(tl.x, a.n_experts, a.status) && in_bounds(tl.z - 1, NMAX, a.status) &&
                    in_bounds(tl.y, a.n_pairs, a.status) && in_bounds((long long)tl.y + tl.z - 1, a.n_pairs, a.status);
    if (!ok) tl = make_int4(0, 0, a.n_pairs < 16 ? a.n_pairs : 16, 0);
    return tl;
}

// One row of a 64 x 64 2-bit tile -> fp16 (c - 1.5) s into output chunks
// c_lo..c_hi-1 (columns 8c..8c+7) of a 128-byte swizzled A row.
STRATA_DEV void dequant_row_q2(const uint8_t *wt, int ri, int c_lo, int c_hi, int row, uint8_t *arow) {
    using F = Qn<2>;
    const uint4 cw = *reinterpret_cast<const uint4 *>(wt + F::kRowBytes * ri);
    uint32_t scb = *reinterpret_cast<const uint32_t *>(wt + F::kScaleOffset + 4 * ri);
    const __half2 s01 = *reinterpret_cast<__half2 *>(&scb);
    const __half2 sh0 = __low2half2(s01), sh1 = __high2half2(s01);
    const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
    const uint32_t words8[4] = {cw.x >> 8, cw.y >> 8, cw.z >> 8, cw.w >> 8};
#pragma unroll
    for (int c = 0; c < 8; ++c) {  // output chunk c: columns 8c .. 8c+7
        if (c < c_lo || c >= c_hi) continue;
        const __half2 sc = (c < 4) ? sh0 : sh1;
        // Columns 8c + 2t, 8c + 2t + 1 (step j = c / 2, half s = c % 2)
        // sit in word t at bits 8s + 6 - 2j and 16 + 8s + 6 - 2j. With
        // the exponent that gives bit 6 - 2j the place value 1, the
        // masked pair reads as the exact fp16 values base_j + code
        // (base 16, 64, 256, 1024); subtracting base_j + 1.5 is exact
        // for j < 3 (17.5, 65.5, 257.5), and in two exact steps for
        // j = 3; one multiply by the scale rounds once.
        const int j = c >> 1;
        const uint32_t m = 0x00030003u << (6 - 2 * j);
        const uint32_t g = j == 0 ? 0x4C004C00u : j == 1 ? 0x54005400u : j == 2 ? 0x5C005C00u : 0x64006400u;
        uint32_t out[4];
#pragma unroll
        for (int pr = 0; pr < 4; ++pr) {
            uint32_t v = (((c & 1) ? words8[pr] : words[pr]) & m) | g;
            __half2 h = *reinterpret_cast<__half2 *>(&v);
            if (j < 3) {
                const float off = j == 0 ? 17.5f : j == 1 ? 65.5f : 257.5f;
                h = __hsub2(h, __floats2half2_rn(off, off));
            } else {
                h = __hsub2(__hsub2(h, __floats2half2_rn(1024.f, 1024.f)), __floats2half2_rn(1.5f, 1.5f));
            }
            h = __hmul2(h, sc);  // (c - 1.5) s
            out[pr] = *reinterpret_cast<uint32_t *>(&h);
        }
        *reinterpret_cast<uint4 *>(arow + ((c ^ (row & 7)) << 4)) = make_uint4(out[0], out[1], out[2], out[3]);
    }
}

// The same for a 4-bit tile row: (c - 7.5) s. Column 8c + 2t + h (chunk
// c = 2j + s) sits in word 2t + j/2 at bits 16h + 8(j%2) + 4s; every pair is
// moved to bits 4..7 / 20..23, where the exponent of 64 gives bit 4 the place
// value 1, so it reads as 64 + code; subtracting 71.5 is exact, and one
// multiply by the scale rounds once.
STRATA_DEV void dequant_row_q4(const uint8_t *wt, int ri, int c_lo, int c_hi, int row, uint8_t *arow) {
    using F = Qn<4>;
    // the row's 32 code bytes as two 16-byte loads; rows 4..7 of each group
    // of 8 take the halves in the other order, so 8 lanes hit 32 banks
    const int sw = (ri >> 2) & 1;
    const uint4 q0 = *reinterpret_cast<const uint4 *>(wt + F::kRowBytes * ri + 16 * sw);
    const uint4 q1 = *reinterpret_cast<const uint4 *>(wt + F::kRowBytes * ri + 16 * (sw ^ 1));
    const uint4 lo = sw ? q1 : q0, hi = sw ? q0 : q1;
    const uint32_t words[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
    uint32_t scb = *reinterpret_cast<const uint32_t *>(wt + F::kScaleOffset + 4 * ri);
    const __half2 s01 = *reinterpret_cast<__half2 *>(&scb);
    const __half2 sh0 = __low2half2(s01), sh1 = __high2half2(s01);
    const __half2 off = __floats2half2_rn(71.5f, 71.5f);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        if (c < c_lo || c >= c_hi) continue;
        const __half2 sc = (c < 4) ? sh0 : sh1;
        const int j = c >> 1, sh = 8 * (j & 1) + 4 * (c & 1);  // bit of the pair's low code
        uint32_t out[4];
#pragma unroll
        for (int pr = 0; pr < 4; ++pr) {
            const uint32_t w = words[2 * pr + (j >> 1)];
            const uint32_t at4 = sh >= 4 ? (w >> (sh - 4)) : (w << 4);
            uint32_t v = (at4 & 0x00F000F0u) | 0x54005400u;
            __half2 h = __hsub2(*reinterpret_cast<__half2 *>(&v), off);
            h = __hmul2(h, sc);  // (c - 7.5) s
            out[pr] = *reinterpret_cast<uint32_t *>(&h);
        }
        *reinterpret_cast<uint4 *>(arow + ((c ^ (row & 7)) << 4)) = make_uint4(out[0], out[1], out[2], out[3]);
    }
}

template <int MODE, int BITS>
__global__ void __launch_bounds__(kGemmThreads, 1) k_expert_gemm(const __grid_constant__ TmaMaps maps, GemmArgs a) {
    using L = GLayout<MODE, BITS>;
    constexpr uint32_t TB = L::TILE;
    constexpr int NMAT = L::NMAT, NMAX = L::NMAX, S = L::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full[S], aready[S], empty[S], accfull[2], accempty[2], fin;
    __shared__ uint32_t tmem_base;
    __shared__ int s_abort;

    auto A_at = [&](int st, int mat) { return smem + (size_t)st * L::STAGE + (size_t)mat * L::A_BYTES; };
    auto B_at = [&](int st) { return smem + (size_t)st * L::STAGE + (size_t)NMAT * L::A_BYTES; };
    auto W_at = [&](int st) { return smem + (size_t)st * L::STAGE + (size_t)NMAT * L::A_BYTES + L::B_BYTES; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_items = (*a.n_tiles) * a.panels;
    const int KSTEPS = a.K / 64;

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&aready[i], kDequantWarps);
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
    if (warp == 0 && lane == 0)
        for (int i = 0; i < 5; ++i) prefetch_tmap(&maps.m[i]);
    if (warp == 1) {
        tmem_alloc(&tmem_base, L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = tmem_base;

    if (warp == 0) {
        // ------------------------------------------------ producer
        if (lane == 0) {
            uint32_t it = 0;
            for (int item = blockIdx.x; item < n_items && !*(volatile int *)&s_abort; item += gridDim.x) {
                const int4 tl = tile_at<NMAX>(a, item / a.panels);
                const int panel = item % a.panels;
                const int npad = (tl.z + 15) & ~15;
                const int bsel = npad <= 16 ? 0 : npad <= 32 ? 1 : npad <= 64 ? 2 : npad <= 128 ? 3 : 4;
                const uint32_t brows = 16u << bsel;
                const uint8_t *wsrc = a.blob + (size_t)tl.x * a.ebytes + a.sec_off + (size_t)(2 * panel) * a.tile_panel;
                bool ok = true;
                for (int ks = 0; ks < KSTEPS; ++ks, ++it) {
                    const int st = it % S;
                    const uint32_t ph = (it / S) & 1;
                    if (!mbar_wait(&empty[st], ph ^ 1, a.status, &s_abort)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[st], L::W_BYTES + brows * 128);
                    if (MODE == 0) {  // (gate, up) pairs of the panel's two 64-row halves
                        bulk_g2s(W_at(st), wsrc + (size_t)ks * a.tile_slice, 2 * TB, &full[st]);
                        bulk_g2s(W_at(st) + 2 * TB, wsrc + a.tile_panel + (size_t)ks * a.tile_slice, 2 * TB,
                                 &full[st]);
                    } else {  // the two 64-row tiles of a down panel are adjacent
                        bulk_g2s(W_at(st), wsrc + (size_t)ks * a.tile_slice, 2 * TB, &full[st]);
                    }
                    tma_load_2d(B_at(st), &maps.m[bsel], ks * 64, tl.y, &full[st]);
                }
                if (!ok) break;
            }
            // copies still in flight (only possible after an abort) land before exit
            const uint32_t first = it > (uint32_t)S ? it - S : 0;
            for (uint32_t j = first; j < it; ++j) mbar_wait(&full[j % S], (j / S) & 1, a.status, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t it = 0, li = 0;
            bool ok = true;
            for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x, ++li) {
                const int4 tl = tile_at<NMAX>(a, item / a.panels);
                const int npad = (tl.z + 15) & ~15;
                const uint32_t idesc = umma_idesc_f16(128, npad);
                const int acc = li & 1;
                if (!mbar_wait(&accempty[acc], ((li >> 1) & 1) ^ 1, a.status, &s_abort)) break;
                tc_fence_after();
                const uint32_t dcol = tbase + (uint32_t)(acc * NMAT * NMAX);
                for (int ks = 0; ks < KSTEPS; ++ks, ++it) {
                    const int st = it % S;
                    const uint32_t ph = (it / S) & 1;
                    if (!mbar_wait(&aready[st], ph, a.status, &s_abort) ||
                        !mbar_wait(&full[st], ph, a.status, &s_abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t bdesc = umma_desc_sw128(B_at(st));
#pragma unroll
                    for (int mat = 0; mat < NMAT; ++mat) {
                        const uint64_t adesc = umma_desc_sw128(A_at(st, mat));
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_f16(dcol + mat * NMAX, adesc + 2 * kk, bdesc + 2 * kk, idesc, (ks | kk) ? 1u : 0u);
                    }
                    umma_commit(&empty[st]);
                }
                if (ok) umma_commit(&accfull[acc]);
            }
            umma_commit(&fin);  // every MMA of this thread is complete before tensor memory is freed
            mbar_wait(&fin, 0, a.status, nullptr);
        }
    } else if (warp < 6) {
        // ------------------------------------------------ epilogue
        const int q = warp & 3;
        const int m = 32 * q + lane;
        uint32_t li = 0;
        for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++li) {
            const int4 tl = tile_at<NMAX>(a, item / a.panels);
            const int panel = item % a.panels;
            const int acc = li & 1;
            if (!mbar_wait(&accfull[acc], (li >> 1) & 1, a.status, &s_abort)) break;
            tc_fence_after();
            const uint32_t trow = tbase + ((uint32_t)(32 * q) << 16) + (uint32_t)(acc * NMAT * NMAX);
            const int n = tl.z, p0 = tl.y;
            const int feat = panel * 128 + m;
            for (int c0 = 0; c0 < n; c0 += 16) {
                if (MODE == 0) {
                    float g[16], u[16];
                    tmem_ld16(trow + c0, g);
                    tmem_ld16(trow + NMAX + c0, u);
                    // G, U carry the pair's token scale s; H = silu(G / s) U s = h s^2
                    const float sl = (c0 + (lane & 15) < n) ? a.pair_s[p0 + c0 + (lane & 15)] : 1.f;
                    const bool unit = __all_sync(0xffffffffu, sl == 1.f);  // no token of the chunk scaled
                    const float il = pow2_inverse(sl);
                    tmem_ld_wait();
                    if (unit) {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (c0 + i < n) a.H[(size_t)(p0 + c0 + i) * a.ldo + feat] = __float2half_rn(silu_fast(g[i]) * u[i]);
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const float sc = __shfl_sync(0xffffffffu, sl, i), inv = __shfl_sync(0xffffffffu, il, i);
                            if (c0 + i < n)
                                a.H[(size_t)(p0 + c0 + i) * a.ldo + feat] =
                                    __float2half_rn(silu_fast(g[i] * inv) * u[i] * sc);
                        }
                    }
                } else {
                    float o[16];
                    tmem_ld16(trow + c0, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (c0 + i < n) a.O[(size_t)(p0 + c0 + i) * a.ldo + feat] = __float2half_rn(o[i]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&accempty[acc]);
        }
    } else {
        // ------------------------------------------------ dequant
        const int dt = threadIdx.x - 192;  // 0..255
        const int row = dt & 127, sub = dt >> 7;
        const int mat = (MODE == 0) ? sub : 0;
        const int c_lo = (MODE == 0) ? 0 : 4 * sub, c_hi = (MODE == 0) ? 8 : 4 * sub + 4;
        uint32_t it = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
            for (int ks = 0; ks < KSTEPS; ++ks, ++it) {
                const int st = it % S;
                const uint32_t ph = (it / S) & 1;
                if (!mbar_wait(&full[st], ph, a.status, &s_abort)) {
                    ok = false;
                    break;
                }
                // row r of the 128-row block: tile half r / 64, row r % 64 of that tile
                const uint8_t *wt = W_at(st) + (row >> 6) * (NMAT * TB) + mat * TB;
                uint8_t *arow = A_at(st, mat) + (row >> 3) * 1024 + (row & 7) * 128;
                if constexpr (BITS == 4)
                    dequant_row_q4(wt, row & 63, c_lo, c_hi, row, arow);
                else
                    dequant_row_q2(wt, row & 63, c_lo, c_hi, row, arow);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&aready[st]);
            }
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, L::TMEM_COLS);
    }
}

template <int MODE>
static void launch_gemm(const TmaMaps &maps, const GemmArgs &a, int bits, int num_sms, cudaStream_t st) {
    if (bits == 4)
        k_expert_gemm<MODE, 4><<<num_sms, kGemmThreads, GLayout<MODE, 4>::SMEM, st>>>(maps, a);
    else
        k_expert_gemm<MODE, 2><<<num_sms, kGemmThreads, GLayout<MODE, 2>::SMEM, st>>>(maps, a);
}

template <int MODE, int BITS>
static cudaError_t set_gemm_limit(int max_smem) {
    if ((int)GLayout<MODE, BITS>::SMEM > max_smem) return cudaErrorInvalidValue;
    return cudaFuncSetAttribute(k_expert_gemm<MODE, BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)GLayout<MODE, BITS>::SMEM);
}

cudaError_t init_gemm_attributes(int max_smem) {
    cudaError_t e;
    if ((e = set_gemm_limit<0, 2>(max_smem)) != cudaSuccess) return e;
    if ((e = set_gemm_limit<1, 2>(max_smem)) != cudaSuccess) return e;
    if ((e = set_gemm_limit<0, 4>(max_smem)) != cudaSuccess) return e;
    return set_gemm_limit<1, 4>(max_smem);
}

void launch_expert_gemm1(const Workspace &ws, const uint8_t *blob, const TmaMaps &maps, int max_tiles, int T,
                         const Shape &s, int num_sms, cudaStream_t st) {
    GemmArgs a{};
    a.blob = blob;
    a.ebytes = expert_bytes(s);
    a.sec_off = 0;
    a.tile_panel = expert_strides(s).gu_panel;
    a.tile_slice = expert_strides(s).gu_slice;
    a.K = s.d;
    a.panels = s.f / 128;
    a.ldo = s.f;
    a.tiles = ws.tiles1;
    a.n_tiles = ws.meta + META_N_TILES1;
    a.H = static_cast<__half *>(ws.hbuf);
    a.pair_s = ws.pair_s;
    a.n_experts = s.E;
    a.n_pairs = T * s.k;
    a.status = ws.status;
    (void)max_tiles;
    launch_gemm<0>(maps, a, s.bits, num_sms, st);
}

// y[t] (+)= sum_j w_j O[pair_of(t, j)] / s_t^2: one CTA per token, 8 features
// per thread (O holds W_down h s_t^2, the token's scale squared).
__global__ void __launch_bounds__(256) k_combine(const __half *__restrict__ O, const int *__restrict__ pair_of,
                                                 const float *__restrict__ topk_w, const float *__restrict__ pair_s,
                                                 float *__restrict__ y, int d, int k, int accumulate, int n_pairs,
                                                 uint32_t *status) {
    const int t = blockIdx.x;
    const int *po = pair_of + (size_t)t * k;
    const float *wt = topk_w + (size_t)t * k;
    const float sc = pair_s[checked_index(po[0], n_pairs, 0, status)];  // every pair of the token has its scale
    const float inv2 = pow2_inverse(sc * sc);
    for (int c = threadIdx.x * 8; c < d; c += 256 * 8) {
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.f;
        for (int j = 0; j < k; ++j) {
            if (!in_bounds(po[j], n_pairs, status)) continue;
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(O + (size_t)po[j] * d + c));
            const __half2 *h = reinterpret_cast<const __half2 *>(&v);
            const float w = wt[j] * inv2;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float2 f = __half22float2(h[q]);
                acc[2 * q] = fmaf(w, f.x, acc[2 * q]);
                acc[2 * q + 1] = fmaf(w, f.y, acc[2 * q + 1]);
            }
        }
        float4 *yr = reinterpret_cast<float4 *>(y + (size_t)t * d + c);
        if (accumulate) {
            const float4 p0 = yr[0], p1 = yr[1];
            acc[0] += p0.x; acc[1] += p0.y; acc[2] += p0.z; acc[3] += p0.w;
            acc[4] += p1.x; acc[5] += p1.y; acc[6] += p1.z; acc[7] += p1.w;
        }
        yr[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        yr[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
}

void launch_combine(const Workspace &ws, float *y, bool accumulate, int T, const Shape &s, cudaStream_t st) {
    if (T <= 0) return;
    k_combine<<<T, 256, 0, st>>>(static_cast<const __half *>(ws.xp), ws.pair_of, ws.topk_w, ws.pair_s, y, s.d, s.k,
                                 accumulate ? 1 : 0, T * s.k, ws.status);
}

void launch_expert_gemm2(const Workspace &ws, const uint8_t *blob, float *y, const TmaMaps &maps, int max_tiles, int T,
                         const Shape &s, int num_sms, cudaStream_t st) {
    GemmArgs a{};
    a.blob = blob;
    a.ebytes = expert_bytes(s);
    a.sec_off = down_section_offset(s);
    a.tile_panel = expert_strides(s).dn_panel;
    a.tile_slice = expert_strides(s).dn_slice;
    a.K = s.f;
    a.panels = s.d / 128;
    a.ldo = s.d;
    a.tiles = ws.tiles2;
    a.n_tiles = ws.meta + META_N_TILES2;
    (void)y;
    a.O = static_cast<__half *>(ws.xp);  // the gathered inputs are dead once gate/up has run
    a.n_experts = s.E;
    a.n_pairs = T * s.k;
    a.status = ws.status;
    (void)max_tiles;
    launch_gemm<1>(maps, a, s.bits, num_sms, st);
}

}  // namespace strata
