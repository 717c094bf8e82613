// decode_fused.cu -- the whole layer for 1..16 tokens in ONE persistent,
// cooperative launch (one CTA per SM).
//
// A decode step verifies 1 + up to 3 draft tokens in one 48-layer pass
// ("Strata：把 125B 大模型塞进 12GB 显卡…", 投机解码); every token uses 10
// experts (核心思路). At these sizes the layer is bound by the bytes of the
// selected experts' 2-bit weights, so the kernel keeps that stream busy and
// pays the routing latency once:
//
//   phase 0  every CTA stages x (optionally bf16(RMSNorm) of the fp32
//            residual, the stack glue), computes the router logits of its
//            slice of experts (fp32, one fixed reduction order per row) and
//            zeroes its slice of y; grid barrier.
//   phase 1  every CTA reads all logits and computes, redundantly and
//            identically, the softmax top-k of every token (ties to the lower
//            expert index), the renormalised weights, the per-expert token
//            lists and the active experts (CTA 0 publishes the routing).
//   phase 2  work items (expert, 128-row panel of gate+up, K split), then
//            (expert, 128-row panel of down, K half), dealt round-robin over
//            the CTAs. One warp per CTA issues 1-D bulk copies of the items'
//            packed tiles into a ring of shared-memory buffers; 16 warps
//            decode the 2-bit codes in registers and multiply them with the
//            tokens on the warp-level MMA (16 rows x 8 tokens x 16 columns,
//            fp16 in, fp32 accumulate). Gate/up sums go to global memory; a
//            per-expert counter releases that expert's down items, which form
//            h = silu(g) * u and add w * W_down h into y with fp32 atomics.
//
// Why the warp MMA and not fp32 FMA: on this GPU, fp32 FMA dot products with
// register dequantisation peak at about 2.2 TB/s of weight bytes for one
// token and 1.0 TB/s for four (issue-bound: the multiply-adds per weight grow
// with the tokens); the MMA takes the multiply-adds off the issue slots so
// the stream can run at HBM speed for every token count up to 16. The
// weights never touch shared memory after the copy: the codes are decoded
// straight into MMA fragment registers.
//
// Exactness of the decode: a code c at mantissa bit p of an fp16 whose
// exponent gives that bit the place value 1 is the exact value base_p + c
// (base 16, 64, 256 or 1024), built with one LOP3 per two codes. The MMA
// accumulates sum_k (base_k + c_k) x_k in fp32; subtracting the per-token
// constant Z = sum_k base_k x_k + 1.5 sum_k x_k of each 32-column block and
// multiplying by the block's fp16 scale gives sum_k (c_k - 1.5) s x_k, up to
// fp32 rounding. x (bf16) is exact in fp16 for |x| in [6.1e-5, 65504]; h is
// rounded to fp16 (relative error <= 2^-11).
//
// Every wait (grid barrier, expert counter, copy barrier) is time-bounded;
// on expiry the kernel records a timeout in the status word and unwinds.
#include "common.cuh"
#include "kernels.h"

namespace strata {

constexpr int kFusedComputeWarps = 16;                        // 8 row groups x 2
constexpr int kFusedThreads = (kFusedComputeWarps + 1) * 32;  // + one copy-issue warp
constexpr int kFusedMaxBuf = 8;

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
    int KS;               // gate/up K splits
    int nbuf;
    uint32_t buf_bytes;
    Workspace ws;
};

// fp16 row strides (halves): +8 makes consecutive token rows start 4 banks
// apart, so the 8 rows x 4 column pairs of one B fragment load hit 32 banks
__host__ __device__ inline int hstride(int n) { return n + 8; }

// shared-memory plan, identical on host and device
struct FusedSmem {
    size_t xh, xz, hh, hz, cand, sel_idx, sel_val, sel_w, cnt, off, act, ptok, pslot, pw, scan, bufs, total;
};

__host__ __device__ inline size_t al16(size_t v) { return (v + 15) & ~(size_t)15; }

__host__ __device__ inline FusedSmem fused_plan(int T, int TT, int d, int f, int E, int k, int nbuf,
                                               uint32_t buf_bytes) {
    const int NS = TT <= 8 ? 8 : 16;  // token slots of the MMA n-tiles
    FusedSmem p;
    size_t o = 0;
    p.xh = o;      o = al16(o + (size_t)(T + 1) * hstride(d) * 2);   // + a zero row
    p.xz = o;      o = al16(o + (size_t)(T + 1) * (d / 32) * 4);
    p.hh = o;      o = al16(o + (size_t)NS * hstride(f / 2) * 2);
    p.hz = o;      o = al16(o + (size_t)NS * (f / 64) * 4);
    p.cand = o;    o = al16(o + (size_t)kFusedComputeWarps * k * 8);
    p.sel_idx = o; o = al16(o + (size_t)T * k * 4);
    p.sel_val = o; o = al16(o + (size_t)T * k * 4);
    p.sel_w = o;   o = al16(o + (size_t)T * k * 4);
    p.cnt = o;     o = al16(o + (size_t)E * 4);
    p.off = o;     o = al16(o + (size_t)(E + 1) * 4);
    p.act = o;     o = al16(o + (size_t)E * 4);
    p.ptok = o;    o = al16(o + (size_t)T * k * 4);
    p.pslot = o;   o = al16(o + (size_t)T * k * 4);
    p.pw = o;      o = al16(o + (size_t)T * k * 4);
    p.scan = o;    o = al16(o + 64 * 4);
    o = (o + 127) & ~(size_t)127;
    p.bufs = o;    o += (size_t)nbuf * buf_bytes;
    p.total = o;
    return p;
}

// monotone map of a float to uint32 (+0 and -0 both map to 0x80000000)
STRATA_DEV uint32_t ordered_key(float v) {
    uint32_t u = __float_as_uint(v + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
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
// compute thread takes the same decision (an abort seen by some threads
// only would strand the others at the next barrier).
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

// One 16-row group x one 64-column tile x NT n-tiles of 8 token slots.
//   wg, wg8  : this lane's code word (word t = lane & 3) of rows g and g+8
//   sg, sg8  : the two fp16 block scales of rows g and g+8
//   xb[n]    : fp16 input row of token slot (n*8 + lane/4), at the tile's column 0
//   z0/z1[n] : per-block constants of token slots n*8 + 2t and n*8 + 2t + 1
// out[n][0..3] += (rows g, g+8) x (slots 2t, 2t+1) dot products.
template <int NT>
STRATA_DEV void tile_mma(uint32_t wg, uint32_t wg8, uint32_t sg, uint32_t sg8, const __half *const (&xb)[NT],
                         const float *const (&z0)[NT], const float *const (&z1)[NT], int nt_active,
                         float (&out)[NT][4]) {
    const int t = threadIdx.x & 3;
    const uint32_t v8g = wg >> 8, v8g8 = wg8 >> 8;
    const float2 s_g = __half22float2(*reinterpret_cast<const __half2 *>(&sg));
    const float2 s_g8 = __half22float2(*reinterpret_cast<const __half2 *>(&sg8));
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
            const uint32_t m = 0x00030003u << (6 - 2 * j), g = step_magic(j);
            const uint32_t a[4] = {(wg & m) | g, (wg8 & m) | g, (v8g & m) | g, (v8g8 & m) | g};
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                if (n < nt_active) {
                    const uint32_t b0 = *reinterpret_cast<const uint32_t *>(xb[n] + 16 * j + 2 * t);
                    const uint32_t b1 = *reinterpret_cast<const uint32_t *>(xb[n] + 16 * j + 8 + 2 * t);
                    mma16816(acc[n], a, b0, b1);
                }
            }
        }
        const float sb = blk ? s_g.y : s_g.x, sb8 = blk ? s_g8.y : s_g8.x;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            if (n < nt_active) {
                const float za = z0[n][blk], zb = z1[n][blk];
                out[n][0] = fmaf(sb, acc[n][0] - za, out[n][0]);
                out[n][1] = fmaf(sb, acc[n][1] - zb, out[n][1]);
                out[n][2] = fmaf(sb8, acc[n][2] - za, out[n][2]);
                out[n][3] = fmaf(sb8, acc[n][3] - zb, out[n][3]);
            }
        }
    }
}

// Per-block constant of one staged fp16 row (columns in 64-column tiles):
// z[b] = sum_{16-col steps j of block b} base_j * X_j + 1.5 * X_b.
STRATA_DEV float block_constant(const __half *row, int b) {
    const int j0 = 2 * (b & 1);
    float x0 = 0.f, x1 = 0.f;
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        x0 += __half2float(row[32 * b + c]);
        x1 += __half2float(row[32 * b + 16 + c]);
    }
    return step_base(j0) * x0 + step_base(j0 + 1) * x1 + 1.5f * (x0 + x1);
}

// ------------------------------------------------------------ top-k helpers
// A lane's candidates: KPL (ordered logit, expert) pairs; 0 / 0x7fffffff mark
// an empty slot. `better` orders by logit descending, then index ascending.
STRATA_DEV bool better(uint32_t ka, uint32_t ia, uint32_t kb, uint32_t ib) { return ka > kb || (ka == kb && ia < ib); }

// Local top-k of one warp: each lane sorts its KPL pairs (register bitonic
// network), then k rounds of a warp max over the lanes' heads (REDUX max on
// the key, REDUX min on the index among the lanes holding that key); the
// winning lane pops its head. Writes k (key, expert) pairs, expert -1 when
// the warp has fewer than k candidates.
template <int KPL>
STRATA_DEV void warp_topk(uint32_t (&kk)[KPL], uint32_t (&id)[KPL], int k, uint32_t *ok, int *oid) {
#pragma unroll
    for (int size = 2; size <= KPL; size <<= 1)
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1)
#pragma unroll
            for (int i = 0; i < KPL; ++i) {
                const int j = i ^ stride;
                if (j > i) {
                    const bool desc = (i & size) == 0;
                    const bool sw = desc ? better(kk[j], id[j], kk[i], id[i]) : better(kk[i], id[i], kk[j], id[j]);
                    const uint32_t tk = kk[i], ti = id[i];
                    kk[i] = sw ? kk[j] : tk;
                    id[i] = sw ? id[j] : ti;
                    kk[j] = sw ? tk : kk[j];
                    id[j] = sw ? ti : id[j];
                }
            }
    const int lane = threadIdx.x & 31;
    for (int j = 0; j < k; ++j) {
        const uint32_t m = __reduce_max_sync(0xffffffffu, kk[0]);
        const uint32_t w = __reduce_min_sync(0xffffffffu, (kk[0] == m) ? id[0] : 0x7fffffffu);
        if (lane == 0) {
            ok[j] = m;
            oid[j] = m ? (int)w : -1;
        }
        if (m && id[0] == w) {
#pragma unroll
            for (int i = 0; i + 1 < KPL; ++i) {
                kk[i] = kk[i + 1];
                id[i] = id[i + 1];
            }
            kk[KPL - 1] = 0u;
            id[KPL - 1] = 0x7fffffffu;
        }
    }
}

template <int KPL>
STRATA_DEV void chunk_topk(const float *lpart, const float *bias, int t, int E, int e0, int e1, int k, uint32_t *ok,
                           int *oid) {
    const int lane = threadIdx.x & 31;
    uint32_t kk[KPL], id[KPL];
#pragma unroll
    for (int i = 0; i < KPL; ++i) {
        kk[i] = 0u;
        id[i] = 0x7fffffffu;
        const int e = e0 + lane + 32 * i;
        if (e < e1) {
            const float4 pq = __ldcg(reinterpret_cast<const float4 *>(lpart + ((size_t)t * E + e) * 4));
            float l = ((pq.x + pq.y) + pq.z) + pq.w;  // fixed order over the K quarters
            if (bias) l += bias[e];
            kk[i] = ordered_key(l);
            id[i] = (uint32_t)e;
        }
    }
    warp_topk<KPL>(kk, id, k, ok, oid);
}

template <int TT>
__global__ void __launch_bounds__(kFusedThreads, 1) k_decode_fused(const FusedArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t full[kFusedMaxBuf], empty[kFusedMaxBuf], wbar;
    __shared__ int s_abort;
    __shared__ float s_red[kFusedComputeWarps][2];
    constexpr int NT = TT <= 8 ? 1 : 2;  // MMA n-tiles of 8 token slots

    const int T = a.T, d = a.d, f = a.f, E = a.E, k = a.k;
    const int FH = f / 2, dpx = hstride(d), dph = hstride(FH);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool producer = warp == kFusedComputeWarps;
    const int G = gridDim.x, b = blockIdx.x;
    const FusedSmem sp = fused_plan(T, TT, d, f, E, k, a.nbuf, a.buf_bytes);
    __half *xh = reinterpret_cast<__half *>(smem + sp.xh);
    float *xz = reinterpret_cast<float *>(smem + sp.xz);
    __half *hh = reinterpret_cast<__half *>(smem + sp.hh);
    float *hz = reinterpret_cast<float *>(smem + sp.hz);
    uint32_t *cand_k = reinterpret_cast<uint32_t *>(smem + sp.cand);
    int *cand_i = reinterpret_cast<int *>(smem + sp.cand) + kFusedComputeWarps * k;
    int *sel_idx = reinterpret_cast<int *>(smem + sp.sel_idx);
    float *sel_val = reinterpret_cast<float *>(smem + sp.sel_val);
    float *sel_w = reinterpret_cast<float *>(smem + sp.sel_w);
    int *cnt = reinterpret_cast<int *>(smem + sp.cnt);
    int *off = reinterpret_cast<int *>(smem + sp.off);
    int *act = reinterpret_cast<int *>(smem + sp.act);
    int *ptok = reinterpret_cast<int *>(smem + sp.ptok);
    int *pslot = reinterpret_cast<int *>(smem + sp.pslot);
    float *pw = reinterpret_cast<float *>(smem + sp.pw);
    int *scan = reinterpret_cast<int *>(smem + sp.scan);
    uint8_t *bufs = smem + sp.bufs;
    float *lpart = a.ws.lpart;  // router partial sums [T][E][4]
    uint32_t *sync = a.ws.sync;  // [0] grid barrier, [1] exit count, [2..2+E) per-expert gate/up counters
    uint32_t *status = a.ws.status;

    // ---------------------------------------------------------------- phase 0
    const int r0 = (int)((long long)E * b / G), r1 = (int)((long long)E * (b + 1) / G);
    const int nr = r1 - r0;
    const uint32_t wbytes = (uint32_t)nr * d * 4;
    const bool wstaged = nr > 0 && wbytes <= (uint32_t)a.nbuf * a.buf_bytes;
    if (producer && lane == 0) {
        for (int i = 0; i < a.nbuf; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kFusedComputeWarps);
        }
        mbar_init(&wbar, 1);
        s_abort = 0;
        fence_mbar_init();
        if (wstaged) {  // this CTA's router rows, one bulk copy
            mbar_arrive_expect_tx(&wbar, wbytes);
            bulk_g2s(bufs, a.W + (size_t)r0 * d, wbytes, &wbar);
        }
    }
    __syncthreads();
    if (!producer) {
        if (a.rms) {  // stack glue: bf16(RMSNorm(x)) of the fp32 residual
            for (int t = 0; t < T; ++t) {
                const float *xr = static_cast<const float *>(a.x) + (size_t)t * d;
                float ss = 0.f;
                for (int c = tid; c < d; c += 512) ss = fmaf(xr[c], xr[c], ss);
                ss = warp_sum(ss);
                if (lane == 0) s_red[warp][t & 1] = ss;
                compute_sync();
                float tot = 0.f;
#pragma unroll
                for (int w2 = 0; w2 < kFusedComputeWarps; ++w2) tot += s_red[w2][t & 1];
                const float inv = 1.0f / sqrtf(tot / (float)d + a.eps);
                for (int c = tid; c < d; c += 512)
                    xh[(size_t)t * dpx + c] = __float2half_rn(__bfloat162float(__float2bfloat16_rn(xr[c] * inv)));
            }
        } else {
            const uint4 *xv = static_cast<const uint4 *>(a.x);
            for (int i = tid; i < T * d / 8; i += 512) {
                const uint4 v = __ldg(xv + i);
                const int t = (i * 8) / d, c = (i * 8) % d;
                const uint32_t u4[4] = {v.x, v.y, v.z, v.w};
                uint32_t h4[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const __half2 hv =
                        __floats2half2_rn(__uint_as_float(u4[j] << 16), __uint_as_float(u4[j] & 0xffff0000u));
                    h4[j] = *reinterpret_cast<const uint32_t *>(&hv);
                }
                *reinterpret_cast<uint4 *>(xh + (size_t)t * dpx + c) = make_uint4(h4[0], h4[1], h4[2], h4[3]);
            }
        }
        for (int c = tid; c < d; c += 512) xh[(size_t)T * dpx + c] = __float2half_rn(0.f);  // zero row
        if (!a.accumulate && !a.rms) {  // zero this CTA's slice of y
            const size_t n = (size_t)T * d, lo = n * b / G, hi = n * (b + 1) / G;
            for (size_t i = lo + tid; i < hi; i += 512) a.y[i] = 0.f;
        }
        compute_sync();
        for (int i = tid; i < (T + 1) * (d / 32); i += 512)  // per-block constants of x
            xz[i] = block_constant(xh + (size_t)(i / (d / 32)) * dpx, i % (d / 32));
        if (wstaged) mbar_wait(&wbar, 0, status, &s_abort);
        const int q4 = d / 4;  // router: warp -> (row, quarter of K), partial sums
        for (int u = warp; u < nr * 4 && !s_abort; u += kFusedComputeWarps) {
            const int rr = u / 4, kq = u % 4;
            const float4 *w4 = wstaged ? reinterpret_cast<const float4 *>(bufs + ((size_t)rr * d + (size_t)kq * q4) * 4)
                                       : reinterpret_cast<const float4 *>(a.W + (size_t)(r0 + rr) * d + (size_t)kq * q4);
            float acc[TT];
#pragma unroll
            for (int t = 0; t < TT; ++t) acc[t] = 0.f;
            for (int i = lane; i < q4 / 4; i += 32) {
                const float4 wv = w4[i];
                const int c = kq * q4 + 4 * i;
#pragma unroll
                for (int t = 0; t < TT; ++t) {
                    if (t < T) {
                        const __half2 *xp = reinterpret_cast<const __half2 *>(xh + (size_t)t * dpx + c);
                        const float2 x01 = __half22float2(xp[0]), x23 = __half22float2(xp[1]);
                        acc[t] = fmaf(wv.x, x01.x, acc[t]);
                        acc[t] = fmaf(wv.y, x01.y, acc[t]);
                        acc[t] = fmaf(wv.z, x23.x, acc[t]);
                        acc[t] = fmaf(wv.w, x23.y, acc[t]);
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < TT; ++t) {
                const float v = warp_sum(acc[t]);
                if (lane == 0 && t < T) lpart[((size_t)t * E + r0 + rr) * 4 + kq] = v;
            }
        }
    }
    __syncthreads();
    if (tid == 0) {  // grid barrier (release our partial logits, acquire everyone's)
        __threadfence();
        atomicAdd(&sync[0], 1u);
        wait_counter(&sync[0], (uint32_t)G, status, &s_abort);
    }
    __syncthreads();

    // ---------------------------------------------------------------- phase 1
    if (!s_abort && !producer) {
        const int wpt = T <= 4 ? 4 : T <= 8 ? 2 : 1;  // warps per token
        const int chunk = (E + wpt - 1) / wpt;
        const int need = (chunk + 31) / 32;  // candidates per lane
        for (int u = warp; u < T * wpt; u += kFusedComputeWarps) {
            const int t = u / wpt, part = u % wpt;
            const int e0 = part * chunk, e1 = min(E, e0 + chunk);
            uint32_t *ok = cand_k + (size_t)u * k;
            int *oi = cand_i + (size_t)u * k;
            if (TT < 16) {
                if (need <= 4) chunk_topk<4>(lpart, a.bias, t, E, e0, e1, k, ok, oi);
                else chunk_topk<8>(lpart, a.bias, t, E, e0, e1, k, ok, oi);
            } else {
                if (need <= 8) chunk_topk<8>(lpart, a.bias, t, E, e0, e1, k, ok, oi);
                else if (need <= 16) chunk_topk<16>(lpart, a.bias, t, E, e0, e1, k, ok, oi);
                else chunk_topk<32>(lpart, a.bias, t, E, e0, e1, k, ok, oi);
            }
        }
        compute_sync();
        const int nc = wpt * k;  // merge: rank of each candidate among its token's candidates
        for (int c = tid; c < T * nc; c += 512) {
            const int t = c / nc;
            if (cand_i[c] < 0) continue;
            const uint32_t kc = cand_k[c], ic = (uint32_t)cand_i[c];
            int rank = 0;
            for (int c2 = t * nc; c2 < (t + 1) * nc; ++c2)
                rank += cand_i[c2] >= 0 && better(cand_k[c2], (uint32_t)cand_i[c2], kc, ic);
            if (rank < k) {
                sel_idx[t * k + rank] = (int)ic;
                sel_val[t * k + rank] = __uint_as_float((kc & 0x80000000u) ? (kc & 0x7FFFFFFFu) : ~kc);
            }
        }
        compute_sync();
        for (int i = tid; i < T * k; i += 512) {  // renormalised softmax weights
            const int t = i / k;
            const float vmax = sel_val[t * k];
            float den = 0.f;
            for (int j = 0; j < k; ++j) den += expf(sel_val[t * k + j] - vmax);
            sel_w[i] = expf(sel_val[i] - vmax) / den;
        }
        for (int e = tid; e < E; e += 512) {  // per-expert counts
            int c = 0;
            for (int i = 0; i < T * k; ++i) c += (sel_idx[i] == e);
            cnt[e] = c;
        }
        compute_sync();
        {  // exclusive scans of the counts and of (count > 0), 2 experts per thread
            const int e0 = 2 * tid;
            const int c0 = e0 < E ? cnt[e0] : 0, c1 = e0 + 1 < E ? cnt[e0 + 1] : 0;
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
                off[e0] = ic;
                if (a0) act[ia] = e0;
            }
            if (e0 + 1 < E) {
                off[e0 + 1] = ic + c0;
                if (a1) act[ia + a0] = e0 + 1;
            }
            if (tid == 0) off[E] = scan[kFusedComputeWarps - 1];
        }
        compute_sync();
        for (int p = tid; p < T * k; p += 512) {  // pairs in (expert, ascending token) order
            const int t = p / k, j = p % k, e = sel_idx[p];
            int rank = 0;
            for (int i = 0; i < t * k; ++i) rank += (sel_idx[i] == e);
            const int pos = off[e] + rank;
            ptok[pos] = t;
            pslot[pos] = j;
            pw[pos] = sel_w[p];
            if (b == 0) a.ws.pair_of[p] = pos;
        }
        compute_sync();
        if (b == 0) {  // publish the routing of this call
            for (int i = tid; i < T * k; i += 512) {
                a.ws.topk_idx[i] = sel_idx[i];
                a.ws.topk_w[i] = sel_w[i];
                a.ws.token_list[i] = ptok[i];
                a.ws.pair_slot[i] = pslot[i];
                a.ws.pair_w[i] = pw[i];
            }
            for (int e = tid; e <= E; e += 512) a.ws.offsets[e] = off[e];
            for (int e = tid; e < E; e += 512) a.ws.counts[e] = cnt[e];
            if (tid == 0) {
                a.ws.meta[META_N_ACTIVE] = scan[32 + kFusedComputeWarps - 1];
                a.ws.meta[META_N_TOKENS] = T;
            }
        }
    }
    __syncthreads();
    const int n_act = s_abort ? 0 : scan[32 + kFusedComputeWarps - 1];

    // ---------------------------------------------------------------- phase 2
    const int KS = a.KS, SL = (d / 64) / KS;
    const int P1 = f / 128, P2 = d / 128, SLD = FH / 64;
    const int n_gu = n_act * P1 * KS, n_dn = n_act * P2 * 2, n_all = n_gu + n_dn;
    const int nq = (n_all > b) ? (n_all - b + G - 1) / G : 0;
    const int NPD = kDecMaxT * k;

    if (producer) {
        // ------------------------------------------------ copy issue (one lane)
        if (lane == 0) {
            int q = 0;
            for (; q < nq && !s_abort; ++q) {
                const int it = b + q * G, bi = q % a.nbuf;
                if (q >= a.nbuf && !mbar_wait(&empty[bi], (uint32_t)(((q / a.nbuf) - 1) & 1), status, &s_abort))
                    break;
                const uint8_t *src;
                uint32_t bytes;
                if (it < n_gu) {
                    const int u = it / (P1 * KS), r = it % (P1 * KS), p = r / KS, ks = r % KS;
                    src = a.blob + (size_t)act[u] * a.ebytes + ((size_t)p * (d / 64) + (size_t)ks * SL) * 5120;
                    bytes = (uint32_t)SL * 5120u;
                } else {
                    const int i2 = it - n_gu;
                    const int u = i2 / (P2 * 2), r = i2 % (P2 * 2), p = r / 2, kd = r % 2;
                    src = a.blob + (size_t)act[u] * a.ebytes + a.down_off +
                          ((size_t)p * (f / 64) + (size_t)kd * SLD) * 2560;
                    bytes = (uint32_t)SLD * 2560u;
                }
                mbar_arrive_expect_tx(&full[bi], bytes);
                bulk_g2s(bufs + (size_t)bi * a.buf_bytes, src, bytes, &full[bi]);
            }
            // copies still in flight (only after an abort) land before exit
            for (int j = (q > a.nbuf ? q - a.nbuf : 0); j < q; ++j)
                mbar_wait(&full[j % a.nbuf], (uint32_t)((j / a.nbuf) & 1), status, nullptr);
            if (wstaged && s_abort) mbar_wait(&wbar, 0, status, nullptr);
        }
    } else {
        // ------------------------------------------------ compute warps
        const int t4 = lane & 3, g = lane >> 2;
        const int rg = warp & 7;  // 16-row group of the 128-row panel
        for (int q = 0; q < nq; ++q) {
            const int it = b + q * G, bi = q % a.nbuf;
            const bool is_gu = it < n_gu;
            int u, p, ks = 0, kd = 0;
            if (is_gu) {
                u = it / (P1 * KS);
                const int r = it % (P1 * KS);
                p = r / KS;
                ks = r % KS;
            } else {
                const int i2 = it - n_gu;
                u = i2 / (P2 * 2);
                const int r = i2 % (P2 * 2);
                p = r / 2;
                kd = r % 2;
            }
            const int e = act[u], ecnt = cnt[e], eoff = off[e];
            if (!is_gu) {
                // every gate/up item of this expert has landed its partial sums
                bool bad = false;
                if (tid == 0) bad = !wait_counter(&sync[2 + u], (uint32_t)(P1 * KS), status, &s_abort);
                if (compute_sync_any(bad || s_abort)) break;
                const int NS = NT * 8;
                for (int i = tid; i < NS * FH; i += 512) {  // h = silu(g) * u on this K half, fp16
                    const int ti = i / FH, c = i % FH;
                    float h = 0.f;
                    if (ti < ecnt) {
                        const int col = kd * FH + c;
                        float gs = 0.f, us = 0.f;
                        for (int s2 = 0; s2 < KS; ++s2) {
                            const size_t base = ((size_t)(s2 * NPD + eoff + ti) * 2) * f + col;
                            gs += __ldcg(a.ws.gu_part + base);
                            us += __ldcg(a.ws.gu_part + base + f);
                        }
                        h = silu_f(gs) * us;
                    }
                    hh[(size_t)ti * dph + c] = __float2half_rn(h);
                }
                compute_sync();
                for (int i = tid; i < NS * (FH / 32); i += 512)
                    hz[i] = block_constant(hh + (size_t)(i / (FH / 32)) * dph, i % (FH / 32));
                compute_sync();
            }
            const bool landed = mbar_wait(&full[bi], (uint32_t)((q / a.nbuf) & 1), status, &s_abort);
            if (compute_sync_any(!landed || s_abort)) break;
            const uint8_t *buf = bufs + (size_t)bi * a.buf_bytes;
            const int nta = (ecnt + 7) / 8 < NT ? (ecnt + 7) / 8 : NT;
            const int gr = 16 * rg + g;  // this lane's rows gr and gr + 8 of the panel
            float out[NT][4];
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int i = 0; i < 4; ++i) out[n][i] = 0.f;
            if (is_gu) {
                const int m = warp >> 3;  // 0 gate, 1 up
                const __half *xb[NT];
                const float *z0[NT], *z1[NT];
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    const int sb = 8 * n + g, sa = 8 * n + 2 * t4;
                    const int tb = sb < ecnt ? ptok[eoff + sb] : T;  // T: the zero row
                    const int ta = sa < ecnt ? ptok[eoff + sa] : T, tc = sa + 1 < ecnt ? ptok[eoff + sa + 1] : T;
                    xb[n] = xh + (size_t)tb * dpx;
                    z0[n] = xz + (size_t)ta * (d / 32);
                    z1[n] = xz + (size_t)tc * (d / 32);
                }
                for (int sl = 0; sl < SL; ++sl) {
                    const int col0 = (ks * SL + sl) * 64;
                    const uint8_t *tile = buf + (size_t)sl * 5120 + m * 2560;
                    const uint32_t wg = *reinterpret_cast<const uint32_t *>(tile + 16 * gr + 4 * t4);
                    const uint32_t wg8 = *reinterpret_cast<const uint32_t *>(tile + 16 * (gr + 8) + 4 * t4);
                    const uint32_t sg = *reinterpret_cast<const uint32_t *>(tile + 2048 + 4 * gr);
                    const uint32_t sg8 = *reinterpret_cast<const uint32_t *>(tile + 2048 + 4 * (gr + 8));
                    const __half *xc[NT];
                    const float *zc0[NT], *zc1[NT];
#pragma unroll
                    for (int n = 0; n < NT; ++n) {
                        xc[n] = xb[n] + col0;
                        zc0[n] = z0[n] + col0 / 32;
                        zc1[n] = z1[n] + col0 / 32;
                    }
                    tile_mma<NT>(wg, wg8, sg, sg8, xc, zc0, zc1, nta, out);
                }
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    const int sa = 8 * n + 2 * t4;
                    const size_t col = (size_t)m * f + p * 128 + gr;
                    if (sa < ecnt) {
                        float *dst = a.ws.gu_part + ((size_t)(ks * NPD + eoff + sa) * 2) * f + col;
                        dst[0] = out[n][0];
                        dst[8] = out[n][2];
                    }
                    if (sa + 1 < ecnt) {
                        float *dst = a.ws.gu_part + ((size_t)(ks * NPD + eoff + sa + 1) * 2) * f + col;
                        dst[0] = out[n][1];
                        dst[8] = out[n][3];
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[bi]);  // buffer consumed by this warp
                compute_sync();
                if (tid == 0) {  // release the partial sums of this item
                    __threadfence();
                    atomicAdd(&sync[2 + u], 1u);
                }
            } else {
                const int half = warp >> 3;  // half of the item's K slices
                const __half *xb[NT];
                const float *z0[NT], *z1[NT];
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    xb[n] = hh + (size_t)(8 * n + g) * dph;
                    z0[n] = hz + (size_t)(8 * n + 2 * t4) * (FH / 32);
                    z1[n] = hz + (size_t)(8 * n + 2 * t4 + 1) * (FH / 32);
                }
                const int s_lo = half * ((SLD + 1) / 2), s_hi = min(SLD, s_lo + (SLD + 1) / 2);
                for (int sl = s_lo; sl < s_hi; ++sl) {
                    const uint8_t *tile = buf + (size_t)sl * 2560;
                    const uint32_t wg = *reinterpret_cast<const uint32_t *>(tile + 16 * gr + 4 * t4);
                    const uint32_t wg8 = *reinterpret_cast<const uint32_t *>(tile + 16 * (gr + 8) + 4 * t4);
                    const uint32_t sg = *reinterpret_cast<const uint32_t *>(tile + 2048 + 4 * gr);
                    const uint32_t sg8 = *reinterpret_cast<const uint32_t *>(tile + 2048 + 4 * (gr + 8));
                    const __half *xc[NT];
                    const float *zc0[NT], *zc1[NT];
#pragma unroll
                    for (int n = 0; n < NT; ++n) {
                        xc[n] = xb[n] + sl * 64;
                        zc0[n] = z0[n] + sl * 2;
                        zc1[n] = z1[n] + sl * 2;
                    }
                    tile_mma<NT>(wg, wg8, sg, sg8, xc, zc0, zc1, nta, out);
                }
                if (s_lo < s_hi) {
#pragma unroll
                    for (int n = 0; n < NT; ++n) {
                        const int sa = 8 * n + 2 * t4;
                        const int row = p * 128 + gr;
                        if (sa < ecnt) {
                            float *yr = a.y + (size_t)ptok[eoff + sa] * d + row;
                            atomicAdd(yr, pw[eoff + sa] * out[n][0]);
                            atomicAdd(yr + 8, pw[eoff + sa] * out[n][2]);
                        }
                        if (sa + 1 < ecnt) {
                            float *yr = a.y + (size_t)ptok[eoff + sa + 1] * d + row;
                            atomicAdd(yr, pw[eoff + sa + 1] * out[n][1]);
                            atomicAdd(yr + 8, pw[eoff + sa + 1] * out[n][3]);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[bi]);
            }
        }
    }
    // the last CTA out clears the counters for the next launch
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const uint32_t prev = atomicAdd(&sync[1], 1u);
        if (prev == (uint32_t)G - 1) {
            sync[0] = 0;
            for (int i = 0, n = s_abort ? E : n_act; i < n; ++i) sync[2 + i] = 0;
            __threadfence();
            sync[1] = 0;
        }
    }
}

// ---------------------------------------------------------------- host side
struct FusedConfig {
    int KS, nbuf;
    uint32_t buf_bytes;
    size_t smem;
};

static FusedConfig fused_config(const Shape &s, int T, int max_smem) {
    FusedConfig c;
    const int TT = T <= 1 ? 1 : T <= 4 ? 4 : 16;
    c.KS = 4;
    while (c.KS > 1 && (s.d / 64) % c.KS) c.KS /= 2;
    const uint32_t gu = (uint32_t)((s.d / 64) / c.KS) * 5120u;
    const uint32_t dn = (uint32_t)((s.f / 2) / 64) * 2560u;
    c.buf_bytes = (gu > dn ? gu : dn);
    c.buf_bytes = (c.buf_bytes + 127) & ~127u;
    const FusedSmem base = fused_plan(T, TT, s.d, s.f, s.E, s.k, 0, c.buf_bytes);
    const long long room = (long long)max_smem - 2048 - (long long)base.total;
    c.nbuf = room > 0 ? (int)(room / c.buf_bytes) : 0;
    if (c.nbuf > kFusedMaxBuf) c.nbuf = kFusedMaxBuf;
    c.smem = fused_plan(T, TT, s.d, s.f, s.E, s.k, c.nbuf, c.buf_bytes).total;
    return c;
}

bool decode_fused_supported(const Shape &s, int T, int max_smem) {
    // one candidate scan per lane holds at most 1024 experts per warp; two
    // experts per compute thread in the count scans
    if (T < 1 || T > kDecMaxT || (s.f / 2) % 64 || s.E > 1024) return false;
    return fused_config(s, T, max_smem).nbuf >= 2;
}

cudaError_t init_fused_attributes(int max_smem) {
    cudaError_t e = set_max_dynamic_smem(k_decode_fused<1>, max_smem);
    if (e == cudaSuccess) e = set_max_dynamic_smem(k_decode_fused<4>, max_smem);
    if (e == cudaSuccess) e = set_max_dynamic_smem(k_decode_fused<16>, max_smem);
    return e;
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
    a.KS = c.KS;
    a.nbuf = c.nbuf;
    a.buf_bytes = c.buf_bytes;
    a.ws = ws;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(num_sms);
    cfg.blockDim = dim3(kFusedThreads);
    cfg.dynamicSmemBytes = c.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (ev) cudaEventRecordWithFlags(ev[2], st, cudaEventRecordExternal);
    cudaError_t e;
    if (T <= 1)
        e = cudaLaunchKernelEx(&cfg, k_decode_fused<1>, a);
    else if (T <= 4)
        e = cudaLaunchKernelEx(&cfg, k_decode_fused<4>, a);
    else
        e = cudaLaunchKernelEx(&cfg, k_decode_fused<16>, a);
    if (ev) cudaEventRecordWithFlags(ev[3], st, cudaEventRecordExternal);
    return e;
}

}  // namespace strata
