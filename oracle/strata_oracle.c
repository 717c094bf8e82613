/*
 * strata_oracle.c -- plain, slow, single-threaded CPU oracle of the
 * routed-expert MoE layer with 2-bit block-quantised experts, and of the
 * 4-bit Hadamard-rotated KV-cache codec.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the library calls this file; only the
 * tests, the smoke check and the benchmark's CPU-baseline leg load it. It
 * shares no code, header, table or constant generator with the CUDA path.
 *
 * Every quantity is computed in IEEE double from the exact values of the
 * inputs (bf16 activations, fp32 router weights and bias, 2-bit codes, fp16
 * scales). No blocking, no fusion, no reordering beyond what the definition
 * itself states.
 *
 * Sources of the definition (page title, section):
 *  - "Strata Skill：把 125B MoE 大模型塞进 12GB 显卡的本地推理引擎", 介绍:
 *    the model holds 24,576 small experts and each generated token uses
 *    only 10 of them (top-10 routing).
 *  - "Strata：把 125B 大模型塞进 12GB 显卡，24,576 个专家在内存与 SSD 之间流动",
 *    核心思路 (10 experts per token) and 代码结构 (a router kernel and an MoE
 *    kernel on the GPU).
 *  - "Strata — 8~12GB 显存跑 125B 大模型的本地推理引擎", §5 table (512
 *    experts per layer) and §2 (48 layers).
 *  - The layer's specification fixes what the pages leave open: the router is
 *    a GEMV followed by a softmax over the layer's experts, top-k selection
 *    with ties going to the lower expert index, renormalisation of the k
 *    selected probabilities; each selected expert is a SwiGLU MLP
 *    (h = silu(W_gate x) * (W_up x), o = W_down h); the outputs are combined
 *    with the routing weights. Weights are stored in 32-weight blocks along
 *    the reduction dimension, code c in {0,1,2,3} meaning (c - 1.5) * scale,
 *    one fp16 scale per block. The pages name this format "Q2_0"
 *    ("Strata Skill…", 功能与原则) but do not give its bits.
 *  - The wider levels of the pages' quality ladder (Q2_0, IQ2_XS, IQ3_XXS,
 *    IQ3_S: "Strata：把 125B 大模型塞进 12GB 显卡…", 能跑多快 table) trade memory
 *    for accuracy. Their lattice codebooks are not on the pages; the 4-bit
 *    block format here is the same rule with 4-bit codes: c in {0..15}
 *    meaning (c - 7.5) * scale, one fp16 scale per 32 weights. In general a
 *    b-bit code means c - (2^b - 1) / 2, centred on zero.
 *
 *  - The optional 4-bit KV cache ("Strata：把 125B 大模型塞进 12GB 显卡…",
 *    长上下文 section; its 代码结构 section lists q4/q8 KV kernels): one
 *    Hadamard rotation of each cached key/value vector, then 4-bit rounding,
 *    halving the memory of the default 8-bit cache. The pages give neither
 *    the rotation's normalisation nor the rounding grid. Read here: the
 *    orthonormal Walsh-Hadamard rotation y = H x / sqrt(D) of each head_dim-D
 *    row (D a power of two, H the Sylvester matrix, H[i][j] =
 *    (-1)^popcount(i & j)); 32-value blocks with one fp16 scale
 *    s = fp16(absmax / 7) (saturated at 65504); q = round-half-even of
 *    the exact product y * fp32(1 / s), clamped to [-7, 7], stored as the
 *    nibble q + 8;
 *    decoding inverts:
 *    x = H ((c - 8) s) / sqrt(D), rounded to bf16. Because the codes are
 *    integers decided by floating point, the encoder computes in fp32 in a
 *    fixed order (butterfly stages of stride 1, 2, ..., D/2, then the
 *    product by fp32(1/sqrt(D)), then the block quantiser); the decoder, whose
 *    output is a float, is the fp64 matrix-vector definition.
 *
 * Readings taken where the pages are silent (each also listed in the design
 * notes): the top-k order key is the logit rounded to fp32 (the precision the
 * GPU decides in), descending, ties to the lower index; the router bias, when
 * given, is added to the logit before the softmax; RMSNorm of the stack uses
 * unit weights and eps supplied by the caller; the stack carries the residual
 * in fp32 and feeds the MoE a bf16-rounded RMSNorm output.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- scalars */

/* bf16 bit pattern -> its exact value */
double oracle_bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* IEEE binary16 bit pattern -> its exact value */
double oracle_fp16_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int expo = (h >> 10) & 0x1f;
    int mant = h & 0x3ff;
    double v;
    if (expo == 0)
        v = ldexp((double)mant, -24); /* subnormal: mant * 2^-24 */
    else
        v = ldexp((double)(1024 + mant), expo - 25); /* (1 + mant/1024) 2^(e-15) */
    return sign ? -v : v;
}

/* double -> bf16, one rounding to nearest, ties to even (finite inputs) */
uint16_t oracle_double_to_bf16(double v)
{
    if (v == 0.0)
        return signbit(v) ? 0x8000 : 0x0000;
    int e;
    frexp(v, &e); /* |v| = m 2^e, m in [0.5, 1) */
    if (e < -125)
        e = -125; /* bf16 subnormal range: fixed quantum 2^-133 */
    double q = ldexp(1.0, e - 8); /* 8 significant bits */
    double r = nearbyint(v / q) * q; /* default rounding mode: ties to even */
    float f = (float)r; /* exact: r has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------ format (dequant) */

/* W[r][k] = (c[r][k] - (2^bits - 1) / 2) * scale[r][k/32] (bits 2: c - 1.5,
 * bits 4: c - 7.5); codes one per byte, row-major [rows x K]; scales fp16
 * bits, row-major [rows x K/32]. */
void oracle_dequant(int rows, int K, int bits, const uint8_t *codes, const uint16_t *scales, double *W)
{
    int nb = K / 32;
    double offset = ((double)(1 << bits) - 1.0) / 2.0;
    for (int r = 0; r < rows; ++r)
        for (int k = 0; k < K; ++k) {
            double s = oracle_fp16_to_double(scales[(size_t)r * nb + k / 32]);
            double c = (double)codes[(size_t)r * K + k];
            W[(size_t)r * K + k] = (c - offset) * s;
        }
}

/* Unpack one matrix of the tiled blob written by the library's packer, from
 * the layout the library's header documents: 64-row x 64-column tiles of
 * 1280 bytes; inside a tile, row i's 64 codes occupy bytes 16i..16i+15 as
 * four little-endian 32-bit words W0..W3, column c = 16j + 8s + 2t + h of the
 * tile sitting in word Wt at bit 16h + 8s + 6 - 2j; the row's two fp16
 * scales (columns 0-31, then 32-63) follow at byte 1024 + 4i. Tile (p, s) --
 * rows 64p.., columns 64s.. -- starts at byte p * panel_stride +
 * s * slice_stride (a lone matrix: slice_stride 1280, panel_stride
 * (K/64) * 1280; an expert interleaves and reorders its tiles, see the
 * wrapper). Returns one code per byte and the fp16 scale bits. */
void oracle_unpack_q2_tiled(int rows, int K, const uint8_t *blob, long panel_stride, long slice_stride,
                            uint8_t *codes, uint16_t *scales)
{
    for (int p = 0; p < rows / 64; ++p)
        for (int s = 0; s < K / 64; ++s) {
            const uint8_t *tile = blob + (size_t)p * (size_t)panel_stride + (size_t)s * (size_t)slice_stride;
            for (int i = 0; i < 64; ++i) {
                int r = p * 64 + i;
                for (int c = 0; c < 64; ++c) {
                    int j = c / 16, sh = (c / 8) % 2, t = (c % 8) / 2, h = c % 2;
                    const uint8_t *wp = tile + 16 * i + 4 * t;
                    uint32_t w = (uint32_t)wp[0] | ((uint32_t)wp[1] << 8) |
                                 ((uint32_t)wp[2] << 16) | ((uint32_t)wp[3] << 24);
                    int bit = 16 * h + 8 * sh + 6 - 2 * j;
                    codes[(size_t)r * K + 64 * s + c] = (uint8_t)((w >> bit) & 3u);
                }
                for (int b = 0; b < 2; ++b) {
                    const uint8_t *sp = tile + 1024 + 4 * i + 2 * b;
                    scales[(size_t)r * (K / 32) + 2 * s + b] = (uint16_t)(sp[0] | (sp[1] << 8));
                }
            }
        }
}

/* The 4-bit tiled layout the library's header documents: 64-row x 64-column
 * tiles of 2304 bytes; inside a tile, row i's 64 codes occupy bytes
 * 32i..32i+31 as eight little-endian 32-bit words W0..W7, column
 * c = 16j + 8s + 2t + e of the tile (j < 4, s < 2, t < 4, e < 2) sitting in
 * word W(2t + j/2) at bit 16e + 8(j % 2) + 4s (four bits); the row's two
 * fp16 scales (columns 0-31, then 32-63) follow at byte 2048 + 4i. Tiles are
 * placed as for the 2-bit layout (a lone matrix: slice_stride 2304,
 * panel_stride (K/64) * 2304). */
void oracle_unpack_q4_tiled(int rows, int K, const uint8_t *blob, long panel_stride, long slice_stride,
                            uint8_t *codes, uint16_t *scales)
{
    for (int p = 0; p < rows / 64; ++p)
        for (int s = 0; s < K / 64; ++s) {
            const uint8_t *tile = blob + (size_t)p * (size_t)panel_stride + (size_t)s * (size_t)slice_stride;
            for (int i = 0; i < 64; ++i) {
                int r = p * 64 + i;
                for (int c = 0; c < 64; ++c) {
                    int j = c / 16, sh = (c / 8) % 2, t = (c % 8) / 2, e = c % 2;
                    const uint8_t *wp = tile + 32 * i + 4 * (2 * t + j / 2);
                    uint32_t w = (uint32_t)wp[0] | ((uint32_t)wp[1] << 8) |
                                 ((uint32_t)wp[2] << 16) | ((uint32_t)wp[3] << 24);
                    int bit = 16 * e + 8 * (j % 2) + 4 * sh;
                    codes[(size_t)r * K + 64 * s + c] = (uint8_t)((w >> bit) & 15u);
                }
                for (int b = 0; b < 2; ++b) {
                    const uint8_t *sp = tile + 2048 + 4 * i + 2 * b;
                    scales[(size_t)r * (K / 32) + 2 * s + b] = (uint16_t)(sp[0] | (sp[1] << 8));
                }
            }
        }
}

/* ------------------------------------------------------------- router */

/* logits[t][e] = sum_i W[e][i] x[t][i] (+ bias[e]) */
void oracle_router_logits(int T, int d, int E, const uint16_t *x_bf16, const float *W,
                          const float *bias, double *logits)
{
    for (int t = 0; t < T; ++t)
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int i = 0; i < d; ++i)
                acc += (double)W[(size_t)e * d + i] * oracle_bf16_to_double(x_bf16[(size_t)t * d + i]);
            if (bias)
                acc += (double)bias[e];
            logits[(size_t)t * E + e] = acc;
        }
}

/* ordering used by the brute-force top-k: fp32 logit descending, then
 * expert index ascending */
typedef struct {
    float key;
    int idx;
} oracle_rank_t;

static int oracle_rank_cmp(const void *a, const void *b)
{
    const oracle_rank_t *x = (const oracle_rank_t *)a, *y = (const oracle_rank_t *)b;
    if (x->key > y->key)
        return -1;
    if (x->key < y->key)
        return 1;
    return (x->idx > y->idx) - (x->idx < y->idx);
}

/* Softmax over all E experts, full sort, keep the first k, renormalise:
 *   p_e = exp(l_e - max l) / sum_e' exp(l_e' - max l)
 *   w_j = p_{e_j} / sum_{j'<k} p_{e_j'}
 * idx[t][j] lists the selected experts in rank order. */
void oracle_topk_softmax(int T, int E, int k, const double *logits, int32_t *idx, double *w)
{
    oracle_rank_t *r = (oracle_rank_t *)malloc(sizeof(oracle_rank_t) * (size_t)E);
    double *p = (double *)malloc(sizeof(double) * (size_t)E);
    for (int t = 0; t < T; ++t) {
        const double *l = logits + (size_t)t * E;
        double mx = l[0];
        for (int e = 1; e < E; ++e)
            if (l[e] > mx)
                mx = l[e];
        double z = 0.0;
        for (int e = 0; e < E; ++e) {
            p[e] = exp(l[e] - mx);
            z += p[e];
        }
        for (int e = 0; e < E; ++e) {
            p[e] /= z;
            r[e].key = (float)l[e];
            r[e].idx = e;
        }
        qsort(r, (size_t)E, sizeof(oracle_rank_t), oracle_rank_cmp);
        double ps = 0.0;
        for (int j = 0; j < k; ++j)
            ps += p[r[j].idx];
        for (int j = 0; j < k; ++j) {
            idx[(size_t)t * k + j] = r[j].idx;
            w[(size_t)t * k + j] = p[r[j].idx] / ps;
        }
    }
    free(r);
    free(p);
}

/* Per-expert token lists: offsets[e] = number of (token, slot) pairs routed
 * to experts < e; the pairs of expert e are listed by ascending token (a token
 * selects an expert at most once), with the slot j at which it was chosen. */
void oracle_expert_lists(int T, int E, int k, const int32_t *idx, int32_t *offsets,
                         int32_t *token_list, int32_t *pair_slot)
{
    int n = 0;
    for (int e = 0; e < E; ++e) {
        offsets[e] = n;
        for (int t = 0; t < T; ++t)
            for (int j = 0; j < k; ++j)
                if (idx[(size_t)t * k + j] == e) {
                    token_list[n] = t;
                    pair_slot[n] = j;
                    ++n;
                }
    }
    offsets[E] = n;
}

/* ------------------------------------------------------------- experts */

static double oracle_silu(double g) { return g / (1.0 + exp(-g)); }

/* SwiGLU expert on n tokens: out[t] = W_down (silu(W_gate x_t) * (W_up x_t)).
 * gate/up: [f x d], down: [d x f]; X, out: [n x d]; codes of `bits` bits. */
void oracle_expert_ffn(int d, int f, int n, int bits, const double *X,
                       const uint8_t *gc, const uint16_t *gs,
                       const uint8_t *uc, const uint16_t *us,
                       const uint8_t *dc, const uint16_t *ds, double *out)
{
    double *Wg = (double *)malloc(sizeof(double) * (size_t)f * d);
    double *Wu = (double *)malloc(sizeof(double) * (size_t)f * d);
    double *Wd = (double *)malloc(sizeof(double) * (size_t)d * f);
    double *h = (double *)malloc(sizeof(double) * (size_t)f);
    oracle_dequant(f, d, bits, gc, gs, Wg);
    oracle_dequant(f, d, bits, uc, us, Wu);
    oracle_dequant(d, f, bits, dc, ds, Wd);
    for (int t = 0; t < n; ++t) {
        const double *x = X + (size_t)t * d;
        for (int r = 0; r < f; ++r) {
            double g = 0.0, u = 0.0;
            for (int i = 0; i < d; ++i) {
                g += Wg[(size_t)r * d + i] * x[i];
                u += Wu[(size_t)r * d + i] * x[i];
            }
            h[r] = oracle_silu(g) * u;
        }
        for (int i = 0; i < d; ++i) {
            double o = 0.0;
            for (int r = 0; r < f; ++r)
                o += Wd[(size_t)i * f + r] * h[r];
            out[(size_t)t * d + i] = o;
        }
    }
    free(Wg);
    free(Wu);
    free(Wd);
    free(h);
}

/* Whole layer for small shapes: route every token, run every selected
 * expert on its tokens, y[t] = sum_j w[t][j] * expert_{idx[t][j]}(x_t).
 * Expert e's weights are gc[e], gs[e], ... (pointer arrays of length E). */
void oracle_moe_layer(int T, int d, int f, int E, int k, int bits, const uint16_t *x_bf16,
                      const float *W, const float *bias,
                      const uint8_t *const *gc, const uint16_t *const *gs,
                      const uint8_t *const *uc, const uint16_t *const *us,
                      const uint8_t *const *dc, const uint16_t *const *ds,
                      double *y, int32_t *idx, double *w)
{
    double *logits = (double *)malloc(sizeof(double) * (size_t)T * E);
    double *X = (double *)malloc(sizeof(double) * (size_t)T * d);
    double *o = (double *)malloc(sizeof(double) * (size_t)d);
    oracle_router_logits(T, d, E, x_bf16, W, bias, logits);
    oracle_topk_softmax(T, E, k, logits, idx, w);
    for (size_t i = 0; i < (size_t)T * d; ++i)
        X[i] = oracle_bf16_to_double(x_bf16[i]);
    for (size_t i = 0; i < (size_t)T * d; ++i)
        y[i] = 0.0;
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int e = idx[(size_t)t * k + j];
            oracle_expert_ffn(d, f, 1, bits, X + (size_t)t * d, gc[e], gs[e], uc[e], us[e], dc[e], ds[e], o);
            for (int i = 0; i < d; ++i)
                y[(size_t)t * d + i] += w[(size_t)t * k + j] * o[i];
        }
    free(logits);
    free(X);
    free(o);
}

/* ------------------------------------------------------------- stack glue */

/* RMSNorm with unit weights, rounded to bf16:
 *   out_i = bf16( x_i / sqrt(mean_j x_j^2 + eps) ) */
void oracle_rmsnorm_bf16(int d, const double *x, double eps, uint16_t *out)
{
    double ss = 0.0;
    for (int i = 0; i < d; ++i)
        ss += x[i] * x[i];
    double inv = 1.0 / sqrt(ss / d + eps);
    for (int i = 0; i < d; ++i)
        out[i] = oracle_double_to_bf16(x[i] * inv);
}

/* Residual update of the stack, carried in fp32 as the library does:
 *   x <- fp32(x + y) */
void oracle_residual_add_f32(int n, float *x, const double *y)
{
    for (int i = 0; i < n; ++i)
        x[i] = (float)((double)x[i] + y[i]);
}

/* ------------------------------------------- 4-bit rotated KV-cache codec */

/* fp32 -> IEEE binary16 bits, one rounding to nearest, ties to even; values
 * beyond the largest finite half become infinity. */
uint16_t oracle_float_to_fp16(float f)
{
    uint16_t sign = signbit(f) ? 0x8000 : 0x0000;
    double v = fabs((double)f);
    if (v == 0.0)
        return sign;
    int e;
    frexp(v, &e); /* v = m 2^e, m in [0.5, 1) */
    int qe = e - 11; /* 11 significant bits: quantum 2^(e-11) */
    if (qe < -24)
        qe = -24; /* subnormal range: fixed quantum 2^-24 */
    double n = nearbyint(ldexp(v, -qe)); /* quanta, ties to even */
    if (n >= 2048.0) { /* rounded up into the next binade */
        n /= 2.0;
        qe += 1;
    }
    if (n < 1024.0) /* subnormal (qe == -24) */
        return sign | (uint16_t)n;
    if (qe + 25 >= 31)
        return sign | 0x7c00;
    return sign | (uint16_t)(((qe + 25) << 10) | ((int)n - 1024));
}

/* Sylvester-Hadamard entry H[i][j] = (-1)^popcount(i & j) */
int oracle_hadamard_sign(int i, int j)
{
    int p = 0;
    for (unsigned m = (unsigned)(i & j); m; m >>= 1)
        p ^= (int)(m & 1u);
    return p ? -1 : 1;
}

/* Unnormalised Walsh-Hadamard transform of v[0..D) in place, in fp32: for
 * stride h = 1, 2, ..., D/2 every pair (i, i + h) with bit h of i clear
 * becomes (v_i + v_{i+h}, v_i - v_{i+h}). Exact arithmetic gives H v. */
void oracle_fwht_f32(int D, float *v)
{
    for (int h = 1; h < D; h *= 2)
        for (int i = 0; i < D; ++i)
            if ((i & h) == 0) {
                float a = v[i], b = v[i + h];
                v[i] = a + b;
                v[i + h] = a - b;
            }
}

/* One 32-value block: s = fp16(min(absmax / 7, 65504)), all in fp32;
 * q_i = clamp(rint(y_i * fp32(1 / s)), -7, 7) (q = 0 when s is zero), the
 * product taken exactly and rounded once, to the nearest integer, ties to
 * even; code q_i + 8. The quotient goes through the fp32 reciprocal of s
 * (the precision the GPU decides in); it differs from an exactly rounded
 * y / s only within a few fp32 ulps of a half-integer. */
void oracle_kv4_quantize_block(const float *y, uint8_t *code, uint16_t *scale_bits)
{
    float amax = 0.0f;
    for (int i = 0; i < 32; ++i)
        if (fabsf(y[i]) > amax)
            amax = fabsf(y[i]);
    float t = amax / 7.0f;
    if (t > 65504.0f)
        t = 65504.0f;
    uint16_t sb = oracle_float_to_fp16(t);
    float s = (float)oracle_fp16_to_double(sb);
    float inv = s > 0.0f ? 1.0f / s : 0.0f;
    for (int i = 0; i < 32; ++i) {
        double r = rint((double)y[i] * (double)inv); /* exact product; ties to even */
        int q = r > 7.0 ? 7 : (r < -7.0 ? -7 : (int)r);
        code[i] = (uint8_t)(q + 8);
    }
    *scale_bits = sb;
}

/* Encoder. x: bf16 bits [rows x D]; codes: [rows x D/2] bytes, element 2j in
 * the low nibble of byte j and 2j+1 in the high nibble; scales: fp16 bits
 * [rows x D/32]. y = fp32(FWHT(x) * fp32(1/sqrt(D))), then the block rule. */
void oracle_kv4_encode(long rows, int D, const uint16_t *x, uint8_t *codes, uint16_t *scales)
{
    float r = (float)(1.0 / sqrt((double)D));
    float *y = malloc((size_t)D * sizeof *y);
    uint8_t q[32];
    for (long row = 0; row < rows; ++row) {
        for (int i = 0; i < D; ++i)
            y[i] = (float)oracle_bf16_to_double(x[(size_t)row * D + i]);
        oracle_fwht_f32(D, y);
        for (int i = 0; i < D; ++i)
            y[i] = y[i] * r;
        for (int b = 0; b < D / 32; ++b) {
            oracle_kv4_quantize_block(y + 32 * b, q, &scales[(size_t)row * (D / 32) + b]);
            for (int j = 0; j < 16; ++j)
                codes[(size_t)row * (D / 2) + 16 * b + j] = (uint8_t)(q[2 * j] | (q[2 * j + 1] << 4));
        }
    }
    free(y);
}

/* Decoder, the definition in double: y_i = (c_i - 8) * s_(i/32),
 * x_j = sum_i H[j][i] y_i / sqrt(D). out: [rows x D] exact-as-double values
 * (the caller rounds them to bf16). */
void oracle_kv4_decode(long rows, int D, const uint8_t *codes, const uint16_t *scales, double *out)
{
    double inv = 1.0 / sqrt((double)D);
    double *y = malloc((size_t)D * sizeof *y);
    for (long row = 0; row < rows; ++row) {
        for (int i = 0; i < D; ++i) {
            int c = (codes[(size_t)row * (D / 2) + i / 2] >> (4 * (i % 2))) & 15;
            y[i] = (c - 8) * oracle_fp16_to_double(scales[(size_t)row * (D / 32) + i / 32]);
        }
        for (int j = 0; j < D; ++j) {
            double acc = 0.0;
            for (int i = 0; i < D; ++i)
                acc += oracle_hadamard_sign(j, i) * y[i];
            out[(size_t)row * D + j] = acc * inv;
        }
    }
    free(y);
}

/* out[i] = bf16(v[i]) for a whole array (one rounding each) */
void oracle_round_bf16_array(long n, const double *v, uint16_t *out)
{
    for (long i = 0; i < n; ++i)
        out[i] = oracle_double_to_bf16(v[i]);
}
