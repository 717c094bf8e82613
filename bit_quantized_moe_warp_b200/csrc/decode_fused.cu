// decode_fused.cu -- the whole layer for 1..16 tokens in ONE persistent,
// cooperative launch (one CTA per SM).
//
// A decode step verifies 1 + up to 3 draft tokens in one 48-layer pass
// ("Strata：把 125B 大模型塞进 12GB 显卡，24,576 个专家在内存与 SSD 之间流动",
// 再快一截：先猜再验的投机解码); every token uses 10 experts (核心思路). At these
// sizes the layer is bound by the bytes of the selected experts' 2-bit (or
// 4-bit) weights and by the latency of the steps before them, so the kernel
// pays the routing latency once and then keeps the weight stream busy. It is
// launched as a programmatic dependent of the previous kernel on the stream
// and waits for it (griddepcontrol.wait) before touching memory.
//
//   phase 0  one warp per CTA starts bulk copies of x and of the CTA's slice
//            of router rows (the bias comes by cp.async); the other warps
//            zero the CTA's slice of y, stage x as fp16 (or bf16(RMSNorm) of
//            the fp32 residual, the stack glue), compute the router partial
//            sums of their rows in K quarters and reduce them, in a fixed
//            order, plus the bias, into the logits; grid barrier, during
//            which the other warps compute the per-block constants of x.
//   phase 1  every CTA reads all logits and computes, redundantly and
//            identically, each token's softmax top-k (logit descending, ties
//            to the lower expert index). The k-th largest of 16 group maxima
//            bounds the token's k-th largest logit from below; the logits at
//            or above it are the candidates, and each candidate's rank is the
//            number of candidates that beat it. Then the renormalised weights
//            and the per-expert token lists (bit masks of tokens, scans over
//            the experts, popcount ranks). The CTA with the least expert work
//            publishes the routing at its end.
//   phase 2  work units (active expert e, 64-row slice p of its hidden
//            layer), dealt round-robin over the CTAs. A unit needs no other
//            unit: it streams the slice's gate and up rows over all of K
//            (contiguous in the blob), forms h = silu(g) * u for the slice in
//            shared memory, then streams the down columns the slice feeds
//            (contiguous too) and adds w * W_down[:, slice] h into y with
//            4-wide fp32 vector reductions. One warp per CTA issues 1-D bulk
//            copies of 40 KB chunks (36 KB of 4-bit tiles) into a ring of
//            shared-memory buffers and
//            asks L2 for chunks other CTAs will copy later (and, while the
//            lists are built, for one unit of the selection per CTA); 16
//            warps decode the codes in registers straight into MMA fragments
//            and multiply on the warp-level MMA (16 rows x 8 tokens x 16
//            columns, fp16 in, fp32 accumulate).
//
// Exactness of the decode: a code c at mantissa bit p of an fp16 whose
// exponent gives that bit the place value 1 is the exact value base_p + c
// (base 16, 64, 256 or 1024), built with one LOP3 per two codes. The MMA
// accumulates sum_k (base_k + c_k) x_k in fp32; subtracting the per-token
// constant Z = sum_k base_k x_k + 1.5 sum_k x_k of each 32-column block and
// multiplying by the block's fp16 scale gives sum_k (c_k - 1.5) s x_k, up to
// fp32 rounding. The 4-bit format (codes 0..15, offset 7.5) moves every
// code to mantissa bits 4..7 (one shift per register at most), so all its
// columns decode as 64 + c and Z = 71.5 sum_k x_k. Each token's x is staged
// as fp16(x * s) with s = 2^e putting its largest |x| in [1, 2): exact for
// every element within 2^-14 of that largest, whatever the token's
// magnitude; the router sums and the gate/up dot products carry s and are
// divided by it exactly. h, which grows as x^2, is rounded to fp16 as h * s^2
// (relative error <= 2^-11) and the down output is divided by s^2.
//
// Every wait (grid barrier, copy barrier) is time-bounded; on expiry the
// kernel records a timeout in the status word and unwinds. Decisions to stop
// are taken at barriers that OR a flag over all compute warps, so no warp is
// left waiting at a barrier that the others skipped.
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "topk.cuh"

namespace strata {

constexpr int kFusedComputeWarps = 16;
// 16 compute warps + one warp that issues the bulk copies, so that copy issue
// and its waits for free ring buffers never hold up a compute warp.
constexpr int kFusedThreads = (kFusedComputeWarps + 1) * 32;
constexpr int kFusedMaxBuf = 16;
// Chunks of 40 KB: every compute warp takes two K slices (or 8 down row
// groups) per chunk, so the fixed cost of a chunk (all warps waking on its
// barrier at once, loading the token fragments) is paid half as often as
// with 20 KB chunks; measured on B200, 4% faster at 1 token, 2.5-4% at 4-16.
// 4-bit tiles (2304 bytes) take 8 K-slices or 16 down tiles per chunk (36 KB).
constexpr uint32_t kChunkBytes = 40960;
template <int BITS>
struct ChunkCfg {
    static constexpr int kTile = Qn<BITS>::kTileBytes;
    static constexpr int kGuSlices = BITS == 4 ? 8 : 16;     // gate/up chunk: K-slices x (gate, up) tiles
    static constexpr int kDownPanels = BITS == 4 ? 16 : 32;  // down chunk: tiles of 64 d-rows
    static_assert(kGuSlices * 2 * kTile <= (int)kChunkBytes && kDownPanels * kTile <= (int)kChunkBytes,
                  "chunk exceeds a ring buffer");
};
constexpr int kHStride = 64 + 8;          // fp16 row stride of h (halves)
constexpr int kRouterRowsMax = 16;        // router rows per CTA (E <= 16 * number of CTAs)
// room left beside the dynamic shared memory for the kernel's static arrays
// (barriers, flags, per-token scales, per-pair weights: about 2.7 KB)
constexpr long long kFusedStaticSmem = 4096;

struct FusedArgs {
    const void *x;        // bf16 [T x d]; fp32 residual [T x d] when rms
    const float *W;       // router [E x d]
    const float *bias;    // [E] or null
    const uint8_t *blob;  // packed experts
    float *y;             // [T x d] (== x when rms)
    int T, d, f, E, k;
    int accumulate;
    int rms;
    float eps;
    size_t ebytes, down_off;
    ExpertStrides xs;
    int nbuf;
    Workspace ws;
};

// fp16 row stride of x (halves): +8 makes consecutive token rows start 4
// banks apart, so the 8 rows x 4 column pairs of one B fragment load hit 32
// different banks
__host__ __device__ inline int hstride(int n) { return n + 8; }

// shared-memory plan, identical on host and device
struct FusedSmem {
    size_t xh, xz, red, hh, hz, lsm, sbias, sel_idx, sel_val, sel_w, gmax, ccnt, mask, prank, cnt, off, act, ptok, pslot,
        pw, scan, bufs, total;
};

// routing candidates kept per token (the selection falls back to an exact
// one-warp pass for a token with more)
constexpr int kCandMax = 64;

__host__ __device__ inline size_t al16(size_t v) { return (v + 15) & ~(size_t)15; }

__host__ __device__ inline int token_slots(int TT) { return TT <= 8 ? 8 : 16; }
// gate/up work split: KSPLIT groups of K slices x (16 / KSPLIT) groups of the
// 8 (matrix, 16-row group) pairs of a 64-row slice; a warp loads a slice's
// token fragments once for all its row groups
__host__ __device__ inline constexpr int gu_ksplit(int TT) { return TT <= 8 ? 8 : 4; }

__host__ __device__ inline FusedSmem fused_plan(int T, int TT, int d, int E, int k, int nbuf) {
    const int NS = token_slots(TT);
    FusedSmem p;
    size_t o = 0;
    p.xh = o;      o = al16(o + (size_t)(T + 1) * hstride(d) * 2);   // + a zero row
    p.xz = o;      o = al16(o + (size_t)(T + 1) * (d / 32) * 4);
    p.red = o;     o = al16(o + (size_t)gu_ksplit(TT) * 2 * 64 * TT * 4);  // [K group][gate/up][row][slot < TT]
    p.hh = o;      o = al16(o + (size_t)NS * kHStride * 2);
    p.hz = o;      o = al16(o + (size_t)NS * 2 * 4);
    p.lsm = o;     o = al16(o + (size_t)T * kRouterRowsMax * 4 * 4);   // router partials [T][row][K quarter]
    p.sbias = o;   o = al16(o + (size_t)kRouterRowsMax * 4);
    p.sel_idx = o; o = al16(o + (size_t)T * k * 4);
    p.sel_val = o; o = al16(o + (size_t)T * k * 4);
    p.sel_w = o;   o = al16(o + (size_t)T * k * 4);
    p.gmax = o;    o = al16(o + (size_t)kDecMaxT * 16 * 4);   // 16 group maxima per token (selection)
    p.ccnt = o;    o = al16(o + (size_t)kDecMaxT * 4);        // candidates per token
    p.mask = o;    o = al16(o + (size_t)E * 4);               // tokens of each expert (bit mask)
    p.prank = o;   o = al16(o + (size_t)T * k * 4);           // sorted position of each pair
    p.cnt = o;     o = al16(o + (size_t)E * 4);
    p.off = o;     o = al16(o + (size_t)(E + 1) * 4);
    p.act = o;     o = al16(o + (size_t)E * 4);
    p.ptok = o;    o = al16(o + (size_t)T * k * 4);
    p.pslot = o;   o = al16(o + (size_t)T * k * 4);
    p.pw = o;      o = al16(o + (size_t)T * k * 4);
    p.scan = o;    o = al16(o + 64 * 4);
    o = (o + 127) & ~(size_t)127;
    p.bufs = o;    o += (size_t)nbuf * kChunkBytes;
    p.total = o;
    return p;
}

// time-bounded spin until *ctr >= target (acquire); false on timeout/abort
STRATA_DEV bool wait_counter(const uint32_t *ctr, uint32_t target, uint32_t *status, volatile int *abort) {
    uint64_t t0 = 0;
    for (uint32_t i = 0;; ++i) {
        uint32_t v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
        if (v >= target) return true;
        if (i == 0) t0 = globaltimer();
        if ((i & 15u) == 15u) {
            if (*abort) return false;
            if (globaltimer() - t0 > kWaitLimitNs) {
                set_status(status, kStatusTimeout);
                *abort = 1;
                return false;
            }
        }
        __nanosleep(32);
    }
}

STRATA_DEV void compute_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kFusedComputeWarps * 32) : "memory"); }

// Barrier of the compute warps that also ORs a flag over them, so that every
// compute thread takes the same decision.
STRATA_DEV bool compute_sync_any(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, 1, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "n"(kFusedComputeWarps * 32)
        : "memory");
    return r != 0;
}

// ------------------------------------------------------------ MMA helpers
STRATA_DEV void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// The 16-column step j of a 64-column tile row keeps its codes at mantissa
// bit p = 6 - 2j; the fp16 exponent gives that bit the place value 1, so the
// decoded value is base_j + c with base_j = 2^(10 - p).
__host__ __device__ constexpr uint32_t step_magic(int j) {
    return j == 0 ? 0x4C004C00u : j == 1 ? 0x54005400u : j == 2 ? 0x5C005C00u : 0x64006400u;
}
__host__ __device__ constexpr float step_base(int j) { return j == 0 ? 16.f : j == 1 ? 64.f : j == 2 ? 256.f : 1024.f; }

// The A-side words of one 16-row group of a tile: lane (g, t) reads, for
// rows g and g+8, word t (2-bit) or words 2t, 2t+1 (4-bit), and the two
// rows' block scales.
template <int BITS>
struct TileRows;
template <>
struct TileRows<2> {
    uint32_t wg, wg8, sg, sg8;
};
template <>
struct TileRows<4> {
    uint2 wg, wg8;
    uint32_t sg, sg8;
};
template <int BITS>
STRATA_DEV TileRows<BITS> load_rows(const uint8_t *tile, int gr) {
    using F = Qn<BITS>;
    const int t = threadIdx.x & 3;
    TileRows<BITS> r;
    if constexpr (BITS == 4) {
        r.wg = *reinterpret_cast<const uint2 *>(tile + F::kRowBytes * gr + 8 * t);
        r.wg8 = *reinterpret_cast<const uint2 *>(tile + F::kRowBytes * (gr + 8) + 8 * t);
    } else {
        r.wg = *reinterpret_cast<const uint32_t *>(tile + F::kRowBytes * gr + 4 * t);
        r.wg8 = *reinterpret_cast<const uint32_t *>(tile + F::kRowBytes * (gr + 8) + 4 * t);
    }
    r.sg = *reinterpret_cast<const uint32_t *>(tile + F::kScaleOffset + 4 * gr);
    r.sg8 = *reinterpret_cast<const uint32_t *>(tile + F::kScaleOffset + 4 * (gr + 8));
    return r;
}

// A fragment of 16-column step j (registers: rows g / g+8 x columns 2t, 2t+1,
// then 2t+8, 2t+9) as exact fp16 values base + code.
// 2-bit: the step's codes sit at mantissa bit 6 - 2j of word t (base 16,
// 64, 256, 1024); the second half (s = 1) is 8 bits higher.
// 4-bit: word 2t + j/2, bits 8(j%2) + 4s: both halves are moved to bits
// 4..7 (base 64).
STRATA_DEV void a_frag(const TileRows<2> &w, int j, uint32_t (&a)[4]) {
    const uint32_t m = 0x00030003u << (6 - 2 * j), g = step_magic(j);
    a[0] = (w.wg & m) | g;
    a[1] = (w.wg8 & m) | g;
    a[2] = ((w.wg >> 8) & m) | g;
    a[3] = ((w.wg8 >> 8) & m) | g;
}
STRATA_DEV void a_frag(const TileRows<4> &w, int j, uint32_t (&a)[4]) {
    constexpr uint32_t m = 0x00F000F0u, g = 0x54005400u;
    const uint32_t x = (j >> 1) ? w.wg.y : w.wg.x, x8 = (j >> 1) ? w.wg8.y : w.wg8.x;
    if (j & 1) {
        a[0] = ((x >> 4) & m) | g;
        a[1] = ((x8 >> 4) & m) | g;
        a[2] = ((x >> 8) & m) | g;
        a[3] = ((x8 >> 8) & m) | g;
    } else {
        a[0] = ((x << 4) & m) | g;
        a[1] = ((x8 << 4) & m) | g;
        a[2] = (x & m) | g;
        a[3] = (x8 & m) | g;
    }
}

// block-constant weight of tile column 2l (and 2l+1): base of its step + the
// format's code offset
template <int BITS>
STRATA_DEV float column_weight(int l) {
    return BITS == 4 ? 71.5f : step_base(l >> 3) + 1.5f;
}

// One 16-row group x one 64-column tile x NT n-tiles of 8 token slots.
// B fragments and block constants come from `bsrc(n, j, b0, b1)` and
// `zsrc(n, blk, z_a, z_b)` (token slots n*8 + 2t and n*8 + 2t + 1).
// out[n][0..3] += (rows g, g+8) x (slots 2t, 2t+1) dot products; with
// ODD false (one token: only slot 0 is real) the odd slots are left alone.
// NT is the number of n-tiles that hold tokens: no per-tile predicate sits
// between the MMAs (it costs about half the loop's throughput).
template <int NT, bool ODD, int BITS, typename BSrc, typename ZSrc>
STRATA_DEV void tile_mma(const TileRows<BITS> &w, BSrc bsrc, ZSrc zsrc, float (&out)[NT][4]) {
    const float2 s_g = __half22float2(*reinterpret_cast<const __half2 *>(&w.sg));
    const float2 s_g8 = __half22float2(*reinterpret_cast<const __half2 *>(&w.sg8));
#pragma unroll
    for (int blk = 0; blk < 2; ++blk) {
        float acc[NT][4];
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[n][i] = 0.f;
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
            const int j = 2 * blk + jj;
            uint32_t a[4];
            a_frag(w, j, a);
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                uint32_t b0, b1;
                bsrc(n, j, b0, b1);
                mma16816(acc[n], a, b0, b1);
            }
        }
        const float sb = blk ? s_g.y : s_g.x, sb8 = blk ? s_g8.y : s_g8.x;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            float za, zb;
            zsrc(n, blk, za, zb);
            out[n][0] = fmaf(sb, acc[n][0] - za, out[n][0]);
            out[n][2] = fmaf(sb8, acc[n][2] - za, out[n][2]);
            if (ODD) {
                out[n][1] = fmaf(sb, acc[n][1] - zb, out[n][1]);
                out[n][3] = fmaf(sb8, acc[n][3] - zb, out[n][3]);
            }
        }
    }
}

// Per-block constants of one staged fp16 row (columns in 64-column tiles),
// one warp: z[b] = sum over the block's columns k of (base(k) + offset) x_k
// (2-bit: sum_j base_j X_j + 1.5 X_b; 4-bit: 71.5 X_b). Lane l reads
// columns 2l, 2l+1 of each tile (step j = l / 8, block l / 16) and the 16
// lanes of a block reduce by shuffles, so the reads are conflict-free; four
// tiles at a time keep four independent shuffle chains in flight.
template <int BITS>
STRATA_DEV void row_block_constants(const __half *row, int ncols, float *z) {
    const int lane = threadIdx.x & 31;
    const float wgt = column_weight<BITS>(lane);
    for (int c0 = 0; c0 < ncols; c0 += 256) {
        float sum[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            sum[q] = 0.f;
            if (c0 + 64 * q < ncols) {
                const float2 v = __half22float2(*reinterpret_cast<const __half2 *>(row + c0 + 64 * q + 2 * lane));
                sum[q] = wgt * (v.x + v.y);
            }
        }
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1)
#pragma unroll
            for (int q = 0; q < 4; ++q) sum[q] += __shfl_xor_sync(0xffffffffu, sum[q], o);
        if ((lane & 15) == 0)
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (c0 + 64 * q < ncols) z[(c0 + 64 * q) / 32 + (lane >> 4)] = sum[q];
    }
}

// One gate/up K slice for the warp's RGM (matrix, row group) pairs: the
// slice's token fragments are loaded once and reused for every pair.
template <int NTA, int NT, int RGM, bool ODD, int BITS>
STRATA_DEV void gu_slice(const uint8_t *tiles, const __half *const (&xb)[NT], const float *const (&z0)[NT],
                         const float *const (&z1)[NT], int col0, int rgm0, int g, float (&out)[RGM][NT][4]) {
    uint32_t bf[NTA][4][2];
    float2 zA[NTA], zB[NTA];
#pragma unroll
    for (int n = 0; n < NTA; ++n) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            bf[n][j][0] = *reinterpret_cast<const uint32_t *>(xb[n] + col0 + 16 * j);
            bf[n][j][1] = *reinterpret_cast<const uint32_t *>(xb[n] + col0 + 16 * j + 8);
        }
        zA[n] = *reinterpret_cast<const float2 *>(z0[n] + col0 / 32);
        zB[n] = ODD ? *reinterpret_cast<const float2 *>(z1[n] + col0 / 32) : zA[n];
    }
#pragma unroll
    for (int r = 0; r < RGM; ++r) {
        const int rgm = rgm0 + r, m = rgm >> 2, gr = 16 * (rgm & 3) + g;
        const TileRows<BITS> w = load_rows<BITS>(tiles + m * Qn<BITS>::kTileBytes, gr);
        tile_mma<NTA, ODD>(
            w,
            [&](int n, int j, uint32_t &b0, uint32_t &b1) {
                b0 = bf[n][j][0];
                b1 = bf[n][j][1];
            },
            [&](int n, int blk, float &za, float &zb) {
                za = blk ? zA[n].y : zA[n].x;
                zb = blk ? zB[n].y : zB[n].x;
            },
            reinterpret_cast<float(&)[NTA][4]>(out[r]));
    }
}

// One down tile row group with h fragments and block constants held in
// registers for the whole unit.
template <int NTA, int NT, bool ODD, int BITS>
STRATA_DEV void down_rows(const TileRows<BITS> &w, const uint32_t (&bf)[NT][4][2], const float (&zf)[NT][2][2],
                          float (&o)[NT][4]) {
    tile_mma<NTA, ODD>(
        w,
        [&](int n, int j, uint32_t &b0, uint32_t &b1) {
            b0 = bf[n][j][0];
            b1 = bf[n][j][1];
        },
        [&](int n, int blk, float &za, float &zb) {
            za = zf[n][blk][0];
            zb = zf[n][blk][1];
        },
        reinterpret_cast<float(&)[NTA][4]>(o));
}

// The exact one-warp selection, kept out of line: it runs only for k > 16 or
// a token with more than kCandMax candidates, and inline its unrolled code
// would sit between the selection's common steps.
__device__ __noinline__ void token_topk_exact(const float *logits, int t, int E, int k, int *sel_idx, float *sel_val) {
    token_topk<16>(logits, t, E, k, sel_idx, sel_val);
}

// Adds the weighted outputs of one 16-row group x 8 token slots (an MMA C
// fragment: lane (g, t) holds rows g, g+8 of slots 2t, 2t+1) into y with
// 4-wide vector reductions. Lanes 4 apart share t; the four lanes of rows
// 4p..4p+3 transpose their values (two butterfly exchanges), after which lane
// 4p + v holds rows 8(v/2) + 4p .. +3 of slot 2t + (v%2), one reduction each:
// a quarter of the scalar atomics, which meet every unit's adds to the same y.
STRATA_DEV void add_rows4(float *y, int d, int row0, const float (&c)[4], int tokA, int tokB, float wA, float wB) {
    const int lane = threadIdx.x & 31, g = lane >> 2;
    float v[4] = {c[0] * wA, c[1] * wB, c[2] * wA, c[3] * wB};  // index 2h + e: row half h, slot parity e
    const bool odd = g & 1, hi = g & 2;
    {  // partner g ^ 1 (lane ^ 4): 2 x 2 transposes
        const float r0 = __shfl_xor_sync(0xffffffffu, odd ? v[0] : v[1], 4);
        const float r1 = __shfl_xor_sync(0xffffffffu, odd ? v[2] : v[3], 4);
        if (odd) {
            v[0] = r0;
            v[2] = r1;
        } else {
            v[1] = r0;
            v[3] = r1;
        }
    }
    {  // partner g ^ 2 (lane ^ 8)
        const float r0 = __shfl_xor_sync(0xffffffffu, hi ? v[0] : v[2], 8);
        const float r1 = __shfl_xor_sync(0xffffffffu, hi ? v[1] : v[3], 8);
        if (hi) {
            v[0] = r0;
            v[1] = r1;
        } else {
            v[2] = r0;
            v[3] = r1;
        }
    }
    const int q = g & 3, tok = (q & 1) ? tokB : tokA;
    if (tok >= 0) {
        float *p = y + (size_t)tok * d + row0 + 8 * (q >> 1) + 4 * (g >> 2);
        asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v[0]), "f"(v[1]), "f"(v[2]),
                     "f"(v[3])
                     : "memory");
    }
}

template <int TT, int BITS>
__global__ void __launch_bounds__(kFusedThreads, 1) k_decode_fused(const FusedArgs a) {
    using CC = ChunkCfg<BITS>;
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t full[kFusedMaxBuf], empty[kFusedMaxBuf], xbar, wbar, selbar;
    __shared__ int s_abort, s_nact;
    // per token: the power-of-two scale s of its staged x and 1 / s (exact);
    // per sorted pair: the routing weight / s^2 of its token
    __shared__ float xsc[kDecMaxT], xin[kDecMaxT], pws[kDecMaxT * 32];
    constexpr int NT = TT <= 8 ? 1 : 2;  // MMA n-tiles of 8 token slots
    constexpr int NS = NT * 8;

    const int T = a.T, d = a.d, f = a.f, E = a.E, k = a.k;
    const int dpx = hstride(d);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool producer = warp == kFusedComputeWarps;
    const int G = gridDim.x, b = blockIdx.x;
    const FusedSmem sp = fused_plan(T, TT, d, E, k, a.nbuf);
    __half *xh = reinterpret_cast<__half *>(smem + sp.xh);
    float *xz = reinterpret_cast<float *>(smem + sp.xz);
    float *red = reinterpret_cast<float *>(smem + sp.red);
    __half *hh = reinterpret_cast<__half *>(smem + sp.hh);
    float *hz = reinterpret_cast<float *>(smem + sp.hz);
    int *sel_idx = reinterpret_cast<int *>(smem + sp.sel_idx);
    float *sel_val = reinterpret_cast<float *>(smem + sp.sel_val);
    float *sel_w = reinterpret_cast<float *>(smem + sp.sel_w);
    uint32_t *gmax = reinterpret_cast<uint32_t *>(smem + sp.gmax);
    int *ccnt = reinterpret_cast<int *>(smem + sp.ccnt);
    uint32_t *mask = reinterpret_cast<uint32_t *>(smem + sp.mask);
    int *prank = reinterpret_cast<int *>(smem + sp.prank);
    int *scan = reinterpret_cast<int *>(smem + sp.scan);
    int *cnt = reinterpret_cast<int *>(smem + sp.cnt);
    int *off = reinterpret_cast<int *>(smem + sp.off);
    int *act = reinterpret_cast<int *>(smem + sp.act);
    int *ptok = reinterpret_cast<int *>(smem + sp.ptok);
    int *pslot = reinterpret_cast<int *>(smem + sp.pslot);
    float *pw = reinterpret_cast<float *>(smem + sp.pw);
    uint8_t *bufs = smem + sp.bufs;
    float *logits = a.ws.lpart;  // router logits [T][E] (+ bias)
    float *lsm = reinterpret_cast<float *>(smem + sp.lsm);
    float *sbias = reinterpret_cast<float *>(smem + sp.sbias);
    uint32_t *sync = a.ws.sync;  // [0] grid barrier, [1] exit count
    uint32_t *status = a.ws.status;

    // ---------------------------------------------------------------- phase 0
    const int r0 = (int)((long long)E * b / G), r1 = (int)((long long)E * (b + 1) / G);
    const int nr = r1 - r0;
    const uint32_t xbytes = (uint32_t)T * d * 2;
    const uint32_t xoff = (xbytes + 127) & ~127u;
    const uint32_t wbytes = (uint32_t)nr * d * 4;
    const uint32_t ring = (uint32_t)a.nbuf * kChunkBytes;
    const bool xstaged = !a.rms && xbytes <= ring;
    const uint32_t woff = xstaged ? xoff : 0u;
    const bool wstaged = nr > 0 && woff + wbytes <= ring;
    // Launched as a dependent of the previous kernel on the stream, this CTA
    // may start while that kernel still runs: only prefetch the router rows
    // into L2 (a hint, harmless whoever writes them), then wait for it to
    // finish before reading or writing anything else.
    if (tid == 0 && nr > 0) prefetch_l2(a.W + (size_t)r0 * d, wbytes);
    griddep_wait();
    griddep_launch_dependents();
    if (warp == kFusedComputeWarps && lane == 0) {
        for (int i = 0; i < a.nbuf; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kFusedComputeWarps);
        }
        mbar_init(&xbar, 1);
        mbar_init(&wbar, 1);
        mbar_init(&selbar, 1);  // the selection is known (phase 1)
        s_abort = 0;
        s_nact = 0;
        fence_mbar_init();
        if (xstaged) {
            mbar_arrive_expect_tx(&xbar, xbytes);
            bulk_g2s(bufs, a.x, xbytes, &xbar);
        }
        if (wstaged) {  // this CTA's router rows, one bulk copy
            mbar_arrive_expect_tx(&wbar, wbytes);
            bulk_g2s(bufs + woff, a.W + (size_t)r0 * d, wbytes, &wbar);
        }
    }
    if (tid < nr) {  // the router bias of this CTA's rows, without waiting for it here
        if (a.bias)
            cp_async4(sbias + tid, a.bias + r0 + tid);
        else
            sbias[tid] = 0.f;
    }
    __syncthreads();
    if (!producer) {
        if (!a.accumulate && !a.rms) {  // zero this CTA's slice of y
            const size_t n = (size_t)T * d, lo = n * b / G, hi = n * (b + 1) / G;
            for (size_t i = lo + tid; i < hi; i += 512) a.y[i] = 0.f;
        }
        if (a.rms) {  // stack glue: bf16(RMSNorm) of the fp32 residual, one warp per token
            for (int t = warp; t < T; t += kFusedComputeWarps) {
                const float4 *xr = reinterpret_cast<const float4 *>(static_cast<const float *>(a.x) + (size_t)t * d);
                float ss = 0.f, am = 0.f;  // sum of squares; largest |x| (for the scale of the normalised row)
                for (int c = lane; c < d / 4; c += 32) {
                    const float4 v = xr[c];
                    ss = fmaf(v.x, v.x, ss);
                    ss = fmaf(v.y, v.y, ss);
                    ss = fmaf(v.z, v.z, ss);
                    ss = fmaf(v.w, v.w, ss);
                    am = fmaxf(am, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
                }
                ss = warp_sum(ss);
                const float inv = 1.0f / sqrtf(ss / (float)d + a.eps);
                am = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(am)));
                const float sc = pow2_scale(am * inv);
                if (lane == 0) {
                    xsc[t] = sc;
                    xin[t] = pow2_inverse(sc);
                }
                for (int c = lane; c < d / 4; c += 32) {
                    const float4 v = xr[c];
                    __half2 *dst = reinterpret_cast<__half2 *>(xh + (size_t)t * dpx + 4 * c);
                    dst[0] = __floats2half2_rn(__bfloat162float(__float2bfloat16_rn(v.x * inv)) * sc,
                                               __bfloat162float(__float2bfloat16_rn(v.y * inv)) * sc);
                    dst[1] = __floats2half2_rn(__bfloat162float(__float2bfloat16_rn(v.z * inv)) * sc,
                                               __bfloat162float(__float2bfloat16_rn(v.w * inv)) * sc);
                }
            }
        } else {
            const uint4 *xv = static_cast<const uint4 *>(a.x);
            if (xstaged) {
                mbar_wait(&xbar, 0, status, &s_abort);
                xv = reinterpret_cast<const uint4 *>(bufs);
            }
            // each token's power-of-two scale (one warp per token: largest |x| from the bf16 bits)
            for (int t = warp; t < T; t += kFusedComputeWarps) {
                uint32_t am = 0u;
                for (int c = lane; c < d / 8; c += 32) {
                    const uint4 v = xv[(size_t)t * (d / 8) + c];
                    const uint32_t u4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) am = max(am, max(u4[j] & 0x7fffu, (u4[j] >> 16) & 0x7fffu));
                }
                am = __reduce_max_sync(0xffffffffu, am);
                if (lane == 0) {
                    const float sc = pow2_scale(__uint_as_float(am << 16));
                    xsc[t] = sc;
                    xin[t] = pow2_inverse(sc);
                }
            }
            compute_sync();
            for (int i = tid; i < T * d / 8; i += 512) {
                const uint4 v = xv[i];
                const int t = (i * 8) / d, c = (i * 8) % d;
                const float sc = xsc[t];
                const uint32_t u4[4] = {v.x, v.y, v.z, v.w};
                uint32_t h4[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const __half2 hv = __floats2half2_rn(__uint_as_float(u4[j] << 16) * sc,
                                                         __uint_as_float(u4[j] & 0xffff0000u) * sc);
                    h4[j] = *reinterpret_cast<const uint32_t *>(&hv);
                }
                *reinterpret_cast<uint4 *>(xh + (size_t)t * dpx + c) = make_uint4(h4[0], h4[1], h4[2], h4[3]);
            }
        }
        for (int c = tid; c < d / 2; c += 512)  // zero row (empty MMA token slots)
            reinterpret_cast<uint32_t *>(xh + (size_t)T * dpx)[c] = 0u;
        compute_sync();
        for (int i = tid; i < d / 32; i += 512) xz[(size_t)T * (d / 32) + i] = 0.f;  // the zero row's constants
        // router: warp -> (row, quarter of K); each lane keeps 16 K-values of
        // W in registers per 512-column step and accumulates every token;
        // the tokens' warp sums run interleaved at the end
        if (wstaged) mbar_wait(&wbar, 0, status, &s_abort);
        const int q4 = d / 4;
        for (int u = warp; u < nr * 4 && !s_abort; u += kFusedComputeWarps) {
            const int rr = u / 4, kq = u % 4;
            const float *wrow = wstaged ? reinterpret_cast<const float *>(bufs + woff) + (size_t)rr * d
                                        : a.W + (size_t)(r0 + rr) * d;
            const int cbase = kq * q4;
            float acc[TT];
#pragma unroll
            for (int t = 0; t < TT; ++t) acc[t] = 0.f;
            for (int c0 = 0; c0 < q4; c0 += 512) {
                const int ncol = min(512, q4 - c0);  // a multiple of 32 (d is a multiple of 128)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    if (128 * i + 4 * lane < ncol) {
                        const float4 wv = *reinterpret_cast<const float4 *>(wrow + cbase + c0 + 128 * i + 4 * lane);
                        // slots past the last token read the zero row: no branch
                        // between the loads, so they are all in flight at once
#pragma unroll
                        for (int t = 0; t < TT; ++t) {
                            const int tr = t < T ? t : T;
                            const uint2 xv =
                                *reinterpret_cast<const uint2 *>(xh + (size_t)tr * dpx + cbase + c0 + 128 * i + 4 * lane);
                            const float2 x01 = __half22float2(*reinterpret_cast<const __half2 *>(&xv.x));
                            const float2 x23 = __half22float2(*reinterpret_cast<const __half2 *>(&xv.y));
                            acc[t] = fmaf(wv.x, x01.x, acc[t]);
                            acc[t] = fmaf(wv.y, x01.y, acc[t]);
                            acc[t] = fmaf(wv.z, x23.x, acc[t]);
                            acc[t] = fmaf(wv.w, x23.y, acc[t]);
                        }
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < TT; ++t)
                if (t < T) acc[t] = warp_sum(acc[t]);
            if (lane == 0)
#pragma unroll
                for (int t = 0; t < TT; ++t)
                    if (t < T) lsm[((size_t)t * kRouterRowsMax + rr) * 4 + kq] = acc[t];
        }
        if (tid < nr) cp_async_wait_all();
        compute_sync();
        for (int i = tid; i < T * nr; i += 512) {  // logits: the K quarters in a fixed order, + bias
            const int t = i / nr, rr = i % nr;
            const float *pq = lsm + ((size_t)t * kRouterRowsMax + rr) * 4;
            // the staged x carries the token's scale s: the sum of the quarters times 1 / s (exact)
            logits[(size_t)t * E + r0 + rr] = ((((pq[0] + pq[1]) + pq[2]) + pq[3]) * xin[t]) + sbias[rr];
        }
    }
    __syncthreads();
    if (tid == 0) {  // grid barrier (release our partial logits, acquire everyone's)
        asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(&sync[0]) : "memory");
        wait_counter(&sync[0], (uint32_t)G, status, &s_abort);
    } else if (!producer && warp > 0) {
        // meanwhile the per-block constants of x (used in phase 2), in pieces
        // of 256 columns of one token over warps 1..15
        const int pieces = (d + 255) / 256;
        for (int u = warp - 1; u < T * pieces; u += kFusedComputeWarps - 1) {
            const int r = u / pieces, c0 = (u % pieces) * 256;
            row_block_constants<BITS>(xh + (size_t)r * dpx + c0, min(256, d - c0), xz + (size_t)r * (d / 32) + c0 / 32);
        }
    }
    __syncthreads();

    // ---------------------------------------------------------------- phase 1
    constexpr int GW = kFusedComputeWarps / TT;  // warps per token in the selection; each takes TT groups
    if (!s_abort && !producer) {
        for (int e = tid; e < E; e += 512) mask[e] = 0u;
        if (tid < kDecMaxT) ccnt[tid] = 0;
        const bool fast = k <= 16;  // the bound needs k group maxima
        const int t = warp / GW, g = warp % GW;
        // Selection, step 1: group q of token t is experts [qE/16, (q+1)E/16)
        // (at most 32); warp (t, g) takes groups g TT .. g TT + TT - 1, one
        // logit of each per lane, and writes their maxima.
        uint32_t key[TT];
        if (fast && t < T) {
            const float *row = logits + (size_t)t * E;
            // every lane loads (past a group's end it re-reads the group's last
            // logit), so the TT loads are in flight at once; then the keys
            float v[TT];
#pragma unroll
            for (int r = 0; r < TT; ++r) {
                const int q = g * TT + r, lo = q * E / 16, hi = (q + 1) * E / 16;
                v[r] = __ldcg(row + (lo + lane < hi ? lo + lane : (hi > lo ? hi - 1 : 0)));
            }
#pragma unroll
            for (int r = 0; r < TT; ++r) {
                const int q = g * TT + r, lo = q * E / 16, hi = (q + 1) * E / 16;
                key[r] = lo + lane < hi ? ordered_key(v[r]) : 0u;  // 0: below every real key
            }
#pragma unroll
            for (int r = 0; r < TT; ++r) {
                const uint32_t m = __reduce_max_sync(0xffffffffu, key[r]);
                if (lane == 0) gmax[t * 16 + g * TT + r] = m;
            }
        }
        compute_sync();
        // Step 2: tau = the k-th largest group maximum; the k maxima at or
        // above it are k distinct logits, so the k-th largest logit is >= tau
        // and every logit >= tau is a candidate (at most kCandMax kept).
        uint2 *cand = reinterpret_cast<uint2 *>(bufs);  // [token][kCandMax] (key, expert); the ring is idle here
        if (fast && t < T) {
            const uint32_t mine = lane < 16 ? gmax[t * 16 + lane] : 0u;
            int rank = 0;
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const uint32_t o = gmax[t * 16 + q];
                rank += (o > mine) || (o == mine && q < lane);
            }
            const uint32_t hit = __ballot_sync(0xffffffffu, lane < 16 && rank == k - 1);
            const uint32_t tau = __shfl_sync(0xffffffffu, mine, __ffs(hit) - 1);
#pragma unroll
            for (int r = 0; r < TT; ++r) {
                const int lo = (g * TT + r) * E / 16;
                const bool c = key[r] != 0u && key[r] >= tau;
                const uint32_t bal = __ballot_sync(0xffffffffu, c);
                if (bal) {
                    int base = 0;
                    if (lane == 0) base = atomicAdd(&ccnt[t], __popc(bal));
                    base = __shfl_sync(0xffffffffu, base, 0);
                    const int pos = base + __popc(bal & ((1u << lane) - 1u));
                    if (c && pos < kCandMax) cand[t * kCandMax + pos] = make_uint2(key[r], (uint32_t)(lo + lane));
                }
            }
        }
        compute_sync();
        // Step 3: a candidate's place is the number of candidates that beat it
        // (larger key, or equal key and lower expert).
        for (int i = tid; i < T * kCandMax; i += 512) {
            const int tt = i / kCandMax, c = i % kCandMax, C = ccnt[tt];
            if (!fast || C > kCandMax || c >= C) continue;
            const uint2 *cl = cand + tt * kCandMax;
            const uint2 me = cl[c];
            int rank = 0;
#pragma unroll 8
            for (int q = 0; q < C; ++q) {
                const uint2 o = cl[q];
                rank += (o.x > me.x) || (o.x == me.x && o.y < me.y);
            }
            if (rank < k) {
                sel_idx[tt * k + rank] = (int)me.y;
                sel_val[tt * k + rank] = key_value(me.x);
            }
        }
        if (warp < T && (!fast || ccnt[warp] > kCandMax))  // exact one-warp selection instead
            token_topk_exact(logits, warp, E, k, sel_idx + warp * k, sel_val + warp * k);
        compute_sync();
        if (tid == 0) mbar_arrive(&selbar);
        // renormalised softmax weights over token t's k selected (k <= 32), on
        // warp 15 - t: warp 0 has just released the selection to the copy warp,
        // and its shuffles measured 0.7 us slower there
        if (kFusedComputeWarps - 1 - warp < T) {
            const int t = kFusedComputeWarps - 1 - warp;
            const float vmax = sel_val[t * k];
            const float ex = lane < k ? expf(sel_val[t * k + lane] - vmax) : 0.f;
            const float den = warp_sum(ex);
            if (lane < k) sel_w[t * k + lane] = ex / den;
        }
        for (int i = tid; i < T * k; i += 512)
            if (in_bounds(sel_idx[i], E, status)) atomicOr(&mask[sel_idx[i]], 1u << (i / k));
        compute_sync();
        {  // counts and exclusive scans of the counts and of (count > 0), 2 experts per thread
            const int e0 = 2 * tid;
            const int c0 = e0 < E ? __popc(mask[e0]) : 0, c1 = e0 + 1 < E ? __popc(mask[e0 + 1]) : 0;
            const int a0 = c0 > 0, a1 = c1 > 0;
            int sc = c0 + c1, sa = a0 + a1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int vc = __shfl_up_sync(0xffffffffu, sc, o), va = __shfl_up_sync(0xffffffffu, sa, o);
                if (lane >= o) {
                    sc += vc;
                    sa += va;
                }
            }
            if (lane == 31) {
                scan[warp] = sc;
                scan[32 + warp] = sa;
            }
            compute_sync();
            if (warp == 0) {
                int vc = lane < kFusedComputeWarps ? scan[lane] : 0;
                int va = lane < kFusedComputeWarps ? scan[32 + lane] : 0;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int uc = __shfl_up_sync(0xffffffffu, vc, o), ua = __shfl_up_sync(0xffffffffu, va, o);
                    if (lane >= o) {
                        vc += uc;
                        va += ua;
                    }
                }
                if (lane < kFusedComputeWarps) {
                    scan[lane] = vc;
                    scan[32 + lane] = va;
                }
            }
            compute_sync();
            const int bc = warp ? scan[warp - 1] : 0, ba = warp ? scan[32 + warp - 1] : 0;
            const int ic = bc + sc - (c0 + c1), ia = ba + sa - (a0 + a1);
            if (e0 < E) {
                cnt[e0] = c0;
                off[e0] = ic;
                if (a0) act[ia] = e0;
            }
            if (e0 + 1 < E) {
                cnt[e0 + 1] = c1;
                off[e0 + 1] = ic + c0;
                if (a1) act[ia + a0] = e0 + 1;
            }
            if (tid == 0) {
                off[E] = scan[kFusedComputeWarps - 1];
                s_nact = scan[32 + kFusedComputeWarps - 1];
            }
        }
        compute_sync();
        for (int p = tid; p < T * k; p += 512) {  // pairs in (expert, ascending token) order
            const int t = p / k, e = sel_idx[p];
            prank[p] = -1;
            if (!in_bounds(e, E, status)) continue;
            const int pos = off[e] + __popc(mask[e] & ((1u << t) - 1u));
            if (!in_bounds(pos, T * k, status)) continue;
            prank[p] = pos;
            ptok[pos] = t;
            pslot[pos] = p % k;
            pw[pos] = sel_w[p];
            pws[pos] = sel_w[p] * xin[t] * xin[t];  // the down products carry s^2 of the token
        }
    } else if (!producer) {
        if (tid == 0) mbar_arrive(&selbar);
    } else if (lane == 0 && mbar_wait(&selbar, 0, status, &s_abort)) {
        // Meanwhile the copy warp asks L2 for one (selected expert, 64-row
        // slice) of the selection per CTA, about two microseconds before the
        // per-expert lists exist and the ring copies start. Up to 4 tokens
        // only: with more, the selection is several waves of units and these
        // requests would queue ahead of the first ring copies.
        const int FP = f / 64, u = b;
        if (TT <= 4 && u < T * k * FP) {
            const int e = sel_idx[u / FP];
            if (in_bounds(e, E, status)) {
                const uint8_t *ebase = a.blob + (size_t)e * a.ebytes;
                const int p = u % FP;
                prefetch_l2(ebase + (size_t)p * a.xs.gu_panel, (uint32_t)(d / 64) * 2u * CC::kTile);
                prefetch_l2(ebase + a.down_off + (size_t)p * a.xs.dn_slice, (uint32_t)(d / 64) * CC::kTile);
            }
        }
    }
    __syncthreads();
    const int n_act = s_abort ? 0 : s_nact;

    // ---------------------------------------------------------------- phase 2
    const int FP = f / 64;   // 64-row slices of the hidden layer
    const int SLK = d / 64;  // K slices of gate/up = 64-row panels of down
    const int nG = (SLK + CC::kGuSlices - 1) / CC::kGuSlices;
    const int nD = (SLK + CC::kDownPanels - 1) / CC::kDownPanels;
    const int n_units = n_act * FP;
    const int nq = (n_units > b) ? (n_units - b + G - 1) / G : 0;
    // chunk i of unit u: its source and size
    auto chunk_src = [&](int u, int i, uint32_t &bytes) -> const uint8_t * {
        const uint8_t *ebase = a.blob + (size_t)checked_index(act[u / FP], E, 0, status) * a.ebytes;
        const int p = u % FP;
        if (i < nG) {
            const int s0 = i * CC::kGuSlices, ns = min(CC::kGuSlices, SLK - s0);
            bytes = (uint32_t)ns * 2u * CC::kTile;
            return ebase + (size_t)p * a.xs.gu_panel + (size_t)s0 * a.xs.gu_slice;
        }
        const int p0 = (i - nG) * CC::kDownPanels, np = min(CC::kDownPanels, SLK - p0);
        bytes = (uint32_t)np * CC::kTile;
        return ebase + a.down_off + (size_t)p * a.xs.dn_slice + (size_t)p0 * a.xs.dn_panel;
    };

    const int per = nG + nD, total = nq * per;
    if (producer) {
        // ------------------------------------------------ copy issue (one lane)
        if (warp == kFusedComputeWarps && lane == 0) {
            fence_proxy_async_smem();  // the staging reads of the ring (phase 0) come before these writes
            int c = 0;
            bool ok = !s_abort;
            for (; c < total && ok; ++c) {
                const int bi = c % a.nbuf;
                if (c >= a.nbuf && !mbar_wait(&empty[bi], (uint32_t)(((c / a.nbuf) - 1) & 1), status, &s_abort)) {
                    ok = false;
                    break;
                }
                uint32_t bytes;
                const uint8_t *src = chunk_src(b + (c / per) * G, c % per, bytes);
                mbar_arrive_expect_tx(&full[bi], bytes);
                bulk_g2s(bufs + (size_t)bi * kChunkBytes, src, bytes, &full[bi]);
                if (c == a.nbuf - 1 || c == total - 1) {
                    // Every CTA, the idle ones too, asks L2 for a share of the
                    // chunks that their owners copy only after their first
                    // ring's worth, so that those copies find their data in L2.
                    for (int ci = b; ci < n_units * per; ci += G) {
                        const int u = ci / per, j = (u / G) * per + ci % per;  // position in the owner's sequence
                        if (j < a.nbuf) continue;
                        uint32_t pb;
                        const uint8_t *ps = chunk_src(u, ci % per, pb);
                        prefetch_l2(ps, pb);
                    }
                }
            }
            if (total == 0)
                for (int ci = b; ci < n_units * per; ci += G) {
                    const int u = ci / per, j = (u / G) * per + ci % per;
                    if (j < a.nbuf) continue;
                    uint32_t pb;
                    const uint8_t *ps = chunk_src(u, ci % per, pb);
                    prefetch_l2(ps, pb);
                }
            // copies still in flight (only after an abort) land before exit
            for (int j = (c > a.nbuf ? c - a.nbuf : 0); j < c; ++j)
                mbar_wait(&full[j % a.nbuf], (uint32_t)((j / a.nbuf) & 1), status, nullptr);
            if (xstaged && s_abort) mbar_wait(&xbar, 0, status, nullptr);
            if (wstaged && s_abort) mbar_wait(&wbar, 0, status, nullptr);
        }
    } else {
        // ------------------------------------------------ compute warps
        constexpr int KSPLIT = gu_ksplit(TT);
        constexpr int RGM = 8 / (kFusedComputeWarps / KSPLIT);  // (matrix, row group) pairs per warp
        constexpr bool ODD = TT > 1;
        const int t4 = lane & 3, g = lane >> 2;
        const int kq = warp % KSPLIT;            // gate/up: K-slice group
        const int rgm0 = (warp / KSPLIT) * RGM;  // gate/up: first (matrix, row group) pair
        int c = 0;
        bool bad = false, stop = false;
        for (int q = 0; q < nq; ++q) {
            const int u = b + q * G;
            const int e = checked_index(act[u / FP], E, 0, status);
            const int ecnt = cnt[e], eoff = off[e];
            const int nta = min((ecnt + 7) / 8, NT);
            // ---- gate / up over all of K
            {
                float out[RGM][NT][4];
#pragma unroll
                for (int r = 0; r < RGM; ++r)
#pragma unroll
                    for (int n = 0; n < NT; ++n)
#pragma unroll
                        for (int i = 0; i < 4; ++i) out[r][n][i] = 0.f;
                const __half *xb[NT];
                const float *z0[NT], *z1[NT];
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    const int sb = 8 * n + g, sa = 8 * n + 2 * t4;
                    // T: the zero row (empty slots; in the checked build also a bad token)
                    xb[n] = xh + (size_t)(sb < ecnt ? checked_index(ptok[eoff + sb], T, T, status) : T) * dpx + 2 * t4;
                    z0[n] = xz + (size_t)(sa < ecnt ? checked_index(ptok[eoff + sa], T, T, status) : T) * (d / 32);
                    z1[n] = xz + (size_t)(sa + 1 < ecnt ? checked_index(ptok[eoff + sa + 1], T, T, status) : T) * (d / 32);
                }
                for (int i = 0; i < nG; ++i, ++c) {
                    const int bi = c % a.nbuf;
                    if (!bad) bad = !mbar_wait(&full[bi], (uint32_t)((c / a.nbuf) & 1), status, &s_abort);
                    if (!bad) {
                        const uint8_t *buf = bufs + (size_t)bi * kChunkBytes;
                        const int s0 = i * CC::kGuSlices, ns = min(CC::kGuSlices, SLK - s0);
                        for (int sl = kq; sl < ns; sl += KSPLIT) {
                            const uint8_t *tiles = buf + (size_t)sl * 2 * CC::kTile;
                            const int col0 = (s0 + sl) * 64;
                            if (NT == 1 || nta == 1)
                                gu_slice<1, NT, RGM, ODD, BITS>(tiles, xb, z0, z1, col0, rgm0, g, out);
                            else
                                gu_slice<NT, NT, RGM, ODD, BITS>(tiles, xb, z0, z1, col0, rgm0, g, out);
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty[bi]);
                }
                if (compute_sync_any(bad || s_abort)) {  // every compute warp takes the same branch
                    stop = true;
                    break;
                }
                // partial sums of this K group: red[kq][matrix][row][slot], slots < TT
#pragma unroll
                for (int r = 0; r < RGM; ++r) {
                    const int rgm = rgm0 + r, m = rgm >> 2, gr = 16 * (rgm & 3) + g;
                    float *rd = red + (size_t)((kq * 2 + m) * 64) * TT;
#pragma unroll
                    for (int n = 0; n < NT; ++n) {
                        const int sa = 8 * n + 2 * t4;
                        if (sa < TT) {
                            rd[gr * TT + sa] = out[r][n][0];
                            rd[(gr + 8) * TT + sa] = out[r][n][2];
                        }
                        if (sa + 1 < TT) {
                            rd[gr * TT + sa + 1] = out[r][n][1];
                            rd[(gr + 8) * TT + sa + 1] = out[r][n][3];
                        }
                    }
                }
            }
            compute_sync();
            // ---- h = silu(g) * u for the slice's 64 rows (fp16) and its block
            // constants: a warp's 32 items are one 32-row block of one slot
            // (NS * 64 is a multiple of 512), reduced with shuffles
            for (int i = tid; i < NS * 64; i += 512) {
                const int slot = i / 64, row = i % 64;
                float h = 0.f;
                if (slot < ecnt) {
                    float gs = 0.f, us = 0.f;
#pragma unroll
                    for (int kg = 0; kg < KSPLIT; ++kg) {
                        gs += red[((kg * 2 + 0) * 64 + row) * TT + slot];
                        us += red[((kg * 2 + 1) * 64 + row) * TT + slot];
                    }
                    // gs, us carry the token's scale s; h = silu(g) u is stored as h s^2
                    // (= silu(gs / s) us s), the down output is divided by s^2
                    const int tk = checked_index(ptok[eoff + slot], T, 0, status);
                    h = silu_fast(gs * xin[tk]) * us * xsc[tk];
                }
                const __half hv = __float2half_rn(h);
                hh[slot * kHStride + row] = hv;
                const float zc = warp_sum(column_weight<BITS>(row >> 1) * __half2float(hv));
                if (lane == 0) hz[slot * 2 + (row >> 5)] = zc;
            }
            compute_sync();
            // ---- down: y[token] += w * W_down[:, slice] h
            {
                uint32_t bf[NT][4][2];
                float zf[NT][2][2];
                int tokA[NT], tokB[NT];
                float wA[NT], wB[NT];
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    const __half *hr = hh + (8 * n + g) * kHStride + 2 * t4;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        bf[n][j][0] = *reinterpret_cast<const uint32_t *>(hr + 16 * j);
                        bf[n][j][1] = *reinterpret_cast<const uint32_t *>(hr + 16 * j + 8);
                    }
                    const int sa = 8 * n + 2 * t4;
#pragma unroll
                    for (int blk = 0; blk < 2; ++blk) {
                        zf[n][blk][0] = hz[sa * 2 + blk];
                        zf[n][blk][1] = hz[(sa + 1) * 2 + blk];
                    }
                    tokA[n] = sa < ecnt ? checked_index(ptok[eoff + sa], T, -1, status) : -1;
                    tokB[n] = sa + 1 < ecnt ? checked_index(ptok[eoff + sa + 1], T, -1, status) : -1;
                    // routing weight / s^2 of the slot's token (h was stored scaled by s^2)
                    wA[n] = sa < ecnt ? pws[eoff + sa] : 0.f;
                    wB[n] = sa + 1 < ecnt ? pws[eoff + sa + 1] : 0.f;
                }
                for (int i = 0; i < nD; ++i, ++c) {
                    const int bi = c % a.nbuf;
                    if (!bad) bad = !mbar_wait(&full[bi], (uint32_t)((c / a.nbuf) & 1), status, &s_abort);
                    if (!bad) {
                        const uint8_t *buf = bufs + (size_t)bi * kChunkBytes;
                        const int p0 = i * CC::kDownPanels, np = min(CC::kDownPanels, SLK - p0);
                        // a warp takes DRG row groups of one panel at once: their rows
                        // are loaded first and their MMA chains run interleaved
                        constexpr int DRG = NT == 1 ? 4 : 2, TPP = 4 / DRG;
                        for (int task = warp; task < np * TPP; task += kFusedComputeWarps) {
                            const int pan = task / TPP, rg0 = (task % TPP) * DRG;
                            TileRows<BITS> w[DRG];
#pragma unroll
                            for (int r = 0; r < DRG; ++r)
                                w[r] = load_rows<BITS>(buf + (size_t)pan * CC::kTile, 16 * (rg0 + r) + g);
                            float o[DRG][NT][4];
#pragma unroll
                            for (int r = 0; r < DRG; ++r)
#pragma unroll
                                for (int n = 0; n < NT; ++n)
#pragma unroll
                                    for (int z = 0; z < 4; ++z) o[r][n][z] = 0.f;
#pragma unroll
                            for (int r = 0; r < DRG; ++r) {
                                if (NT == 1 || nta == 1)
                                    down_rows<1, NT, ODD, BITS>(w[r], bf, zf, o[r]);
                                else
                                    down_rows<NT, NT, ODD, BITS>(w[r], bf, zf, o[r]);
                            }
#pragma unroll
                            for (int r = 0; r < DRG; ++r) {
                                const int row0 = (p0 + pan) * 64 + 16 * (rg0 + r);
#pragma unroll
                                for (int n = 0; n < NT; ++n)
                                    add_rows4(a.y, d, row0, o[r][n], tokA[n], tokB[n], wA[n], wB[n]);
                            }
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty[bi]);
                }
            }
            // a failed copy wait in the down chunks reaches the other warps
            // at the next unit's first barrier, or at the one below
        }
        // Either every compute warp left the loop through the barrier above
        // (stop), or none did and all of them meet here once.
        if (!stop) compute_sync_any(bad);
    }
    __syncthreads();
    if (b == G - 1 && !s_abort) {
        // The routing of this call, published by the CTA dealt the fewest units.
        for (int e = tid; e <= E; e += kFusedThreads) a.ws.offsets[e] = off[e];
        for (int e = tid; e < E; e += kFusedThreads) a.ws.counts[e] = cnt[e];
        if (tid == 0) {
            a.ws.meta[META_N_ACTIVE] = n_act;
            a.ws.meta[META_N_TOKENS] = T;
        }
        for (int i = tid; i < T * k; i += kFusedThreads) {
            a.ws.topk_idx[i] = sel_idx[i];
            a.ws.topk_w[i] = sel_w[i];
            a.ws.token_list[i] = ptok[i];
            a.ws.pair_slot[i] = pslot[i];
            a.ws.pair_w[i] = pw[i];
            a.ws.pair_of[i] = prank[i];
        }
    }
    // the last CTA out clears the counters for the next launch
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const uint32_t prev = atomicAdd(&sync[1], 1u);
        if (prev == (uint32_t)G - 1) {
            sync[0] = 0;
            __threadfence();
            sync[1] = 0;
        }
    }
}

// ---------------------------------------------------------------- host side
struct FusedConfig {
    int nbuf;
    size_t smem;
};

// The ring stays under kFusedSmemSoftCap when that still leaves
// kFusedMinRing chunks, and only otherwise grows to the device limit. The
// cap comes from a B200 microbenchmark of the MMA loop alone, which ran about
// 40% slower when the block's shared memory forced the largest carveout (L1
// left with about 28 KB). In the whole kernel that effect did not show: with
// 40 KB chunks the default shapes take the device limit (3-5 chunks) and run
// faster than 20 KB chunks under the cap, and lower caps measured slower.
constexpr long long kFusedSmemSoftCap = 150 * 1024;
constexpr int kFusedMinRing = 4;

static FusedConfig fused_config(const Shape &s, int T, int max_smem) {
    FusedConfig c;
    const int TT = T <= 1 ? 1 : T <= 4 ? 4 : T <= 8 ? 8 : 16;
    const FusedSmem base = fused_plan(T, TT, s.d, s.E, s.k, 0);
    auto ring = [&](long long limit) {
        const long long room = limit - kFusedStaticSmem - (long long)base.total;
        const int n = room > 0 ? (int)(room / kChunkBytes) : 0;
        return n > kFusedMaxBuf ? kFusedMaxBuf : n;
    };
    c.nbuf = ring(kFusedSmemSoftCap < max_smem ? kFusedSmemSoftCap : max_smem);
    if (c.nbuf < kFusedMinRing) c.nbuf = ring(max_smem);
    c.smem = fused_plan(T, TT, s.d, s.E, s.k, c.nbuf).total;
    return c;
}

bool decode_fused_supported(const Shape &s, int T, int max_smem, int num_sms) {
    // one warp per token in the routing, 16 logits per lane read 4 at a
    // time; at most kRouterRowsMax router rows per CTA; 64-column tiles on
    // both sides of every matrix
    if (T < 1 || T > kDecMaxT || s.E > 512 || s.E % 4 || s.d % 64 || s.f % 64) return false;
    if (num_sms < 1 || (s.E + num_sms - 1) / num_sms > kRouterRowsMax) return false;
    return fused_config(s, T, max_smem).nbuf >= 2;
}

// The kernels' shared-memory limit is raised only as far as the launches
// need: a larger limit makes the driver pick a larger shared-memory carveout
// (less L1), which slows the MMA loops (see kFusedSmemSoftCap). Kept per
// device and instantiation; raised at layer creation, before any capture.
static std::mutex g_limit_mutex;
static int g_limit[64][8];

// the instantiation of a token count and code width
using FusedKernel = void (*)(const FusedArgs);
static FusedKernel kernel_of(int slot) {
    static const FusedKernel k[8] = {k_decode_fused<1, 2>, k_decode_fused<4, 2>, k_decode_fused<8, 2>,
                                     k_decode_fused<16, 2>, k_decode_fused<1, 4>, k_decode_fused<4, 4>,
                                     k_decode_fused<8, 4>, k_decode_fused<16, 4>};
    return k[slot];
}

static cudaError_t ensure_limit(int slot, int need) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_limit_mutex);
    if (g_limit[dev][slot] >= need) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel_of(slot), cudaFuncAttributeMaxDynamicSharedMemorySize, need);
    if (e == cudaSuccess) g_limit[dev][slot] = need;
    return e;
}

static int slot_of(int T, int bits) { return (T <= 1 ? 0 : T <= 4 ? 1 : T <= 8 ? 2 : 3) + (bits == 4 ? 4 : 0); }

cudaError_t init_fused_attributes(const Shape &s, int max_tokens, int max_smem, int num_sms) {
    static const int tts[4] = {1, 4, 8, 16};
    for (int i = 0; i < 4; ++i) {
        const int T = tts[i] < max_tokens ? tts[i] : max_tokens;
        if (slot_of(T, 2) != i || !decode_fused_supported(s, T, max_smem, num_sms)) continue;
        const cudaError_t e = ensure_limit(slot_of(T, s.bits), (int)fused_config(s, T, max_smem).smem);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_decode_fused(const Workspace &ws, const void *x, const float *W, const float *bias,
                                const uint8_t *blob, float *y, bool accumulate, bool rms, float eps, int T,
                                const Shape &s, int num_sms, int max_smem, cudaStream_t st, cudaEvent_t *ev) {
    const FusedConfig c = fused_config(s, T, max_smem);
    FusedArgs a;
    a.x = x;
    a.W = W;
    a.bias = bias;
    a.blob = blob;
    a.y = y;
    a.T = T;
    a.d = s.d;
    a.f = s.f;
    a.E = s.E;
    a.k = s.k;
    a.accumulate = accumulate ? 1 : 0;
    a.rms = rms ? 1 : 0;
    a.eps = eps;
    a.ebytes = expert_bytes(s);
    a.down_off = down_section_offset(s);
    a.xs = expert_strides(s);
    a.nbuf = c.nbuf;
    a.ws = ws;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(num_sms);
    cfg.blockDim = dim3(kFusedThreads);
    cfg.dynamicSmemBytes = c.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    // programmatic dependent launch: this grid is set up while the previous
    // kernel on the stream finishes (the kernel waits for it before its work)
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const int slot = slot_of(T, s.bits);
    cudaError_t e = ensure_limit(slot, (int)c.smem);  // a no-op after layer creation
    if (e != cudaSuccess) return e;
    if (ev) cudaEventRecordWithFlags(ev[2], st, cudaEventRecordExternal);
    e = cudaLaunchKernelEx(&cfg, kernel_of(slot), a);
    if (ev) cudaEventRecordWithFlags(ev[3], st, cudaEventRecordExternal);
    return e;
}

}  // namespace strata
