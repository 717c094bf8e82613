/*
 * strata_kv.h -- C ABI of the 4-bit Hadamard-rotated KV-cache codec.
 *
 * Source: "Strata：把 125B 大模型塞进 12GB 显卡，24,576 个专家在内存与 SSD 之间流动",
 * section 长上下文 (an optional 4-bit KV cache: one Hadamard rotation of the
 * cached vectors, then 4-bit rounding, half the memory of the default 8-bit
 * cache, at some loss of accuracy on long documents) and section 代码结构
 * (the engine's q4/q8 KV kernels). The pages fix neither the rotation's
 * normalisation nor the rounding grid; this library reads them as follows.
 *
 * Format, per row of D values (one key or value head vector of one token;
 * D = head_dim in {64, 128, 256}):
 *   y = H x / sqrt(D), H the D x D Sylvester Hadamard matrix,
 *       H[i][j] = (-1)^popcount(i & j) (an orthonormal rotation);
 *   per block b of 32 consecutive y values: scale s_b = fp16(min(absmax_b / 7,
 *       65504)); code c_i = clamp(rint(y_i * fp32(1 / s_b)), -7, 7) + 8 (rint
 *       rounds half to even; c_i = 8 when s_b is zero);
 *   codes: D/2 bytes per row, value 2j in the low nibble of byte j, value
 *       2j + 1 in the high nibble; scales: D/32 fp16 per row.
 *   Decoding: x'_j = sum_i H[j][i] (c_i - 8) s_(i/32) / sqrt(D), to bf16.
 * The encoder's arithmetic is fp32 in a fixed order: butterfly stages of
 * stride 1, 2, ..., D/2 ((a, b) -> (a + b, a - b)), the product by
 * fp32(1/sqrt(D)), then the block rule above; so the codes and scales are a
 * deterministic function of the input bits. The decoder's output is within
 * fp32 rounding of the exact inverse, then rounded to bf16.
 *
 * Memory: 0.5625 bytes per value (4.5 bits) against 2 for bf16 and 1.0625
 * for an 8-bit cache with the same blocks.
 *
 * Conventions (as in strata_moe.h): every pointer is device memory, rows are
 * contiguous (row r of x at x + r * D, of codes at codes + r * D / 2, of
 * scales at scales + r * D / 32), calls are asynchronous on `stream` and the
 * caller owns every buffer. x and out must be 16-byte aligned, codes 4-byte
 * aligned, scales 2-byte aligned. Inputs must be finite (a NaN or infinity
 * gives unspecified codes, never a fault). n_rows == 0 is a no-op.
 * Errors: STRATA_ERR_INVALID_ARG (NULL pointer with n_rows > 0, n_rows < 0,
 * misalignment), STRATA_ERR_UNSUPPORTED (head_dim not 64, 128 or 256),
 * STRATA_ERR_CUDA (launch failure); the reason is in strata_last_error().
 */
#ifndef STRATA_KV_H
#define STRATA_KV_H

#include "strata_moe.h"

#ifdef __cplusplus
extern "C" {
#endif

#define STRATA_KV4_BLOCK 32

/* Bytes of codes and of scales for n_rows rows of head_dim D. */
size_t strata_kv4_code_bytes(int64_t n_rows, int32_t head_dim);
size_t strata_kv4_scale_bytes(int64_t n_rows, int32_t head_dim);

/* Encode n_rows bf16 rows x [n_rows x head_dim] into codes [n_rows x
 * head_dim/2] and fp16 scales [n_rows x head_dim/32]. Appending to a cache:
 * pass the cache's codes and scales pointers advanced by the first new
 * row. */
strata_status strata_kv4_encode(const void *x, int64_t n_rows, int32_t head_dim, void *codes, void *scales,
                                strata_stream_t stream);

/* Decode codes and scales of n_rows rows into bf16 out [n_rows x head_dim]. */
strata_status strata_kv4_decode(const void *codes, const void *scales, int64_t n_rows, int32_t head_dim, void *out,
                                strata_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* STRATA_KV_H */
