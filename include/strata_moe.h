/*
 * strata_moe.h -- C ABI of the B200 (sm_100a) routed-expert MoE layer with
 * 2-bit block-quantised experts.
 *
 * What the layer computes (sources: the pages' titles and sections):
 *   - "Strata Skill：把 125B MoE 大模型塞进 12GB 显卡的本地推理引擎", 介绍, and
 *     "Strata：把 125B 大模型塞进 12GB 显卡，24,576 个专家在内存与 SSD 之间流动",
 *     核心思路: each token is served by 10 of the layer's experts.
 *   - "Strata — 8~12GB 显存跑 125B 大模型的本地推理引擎", §5 table: 512
 *     experts per layer; §2 and the second page's 投机解码: 48 layers, and a
 *     decode step verifies 1 + up to 3 draft tokens in one 48-layer pass.
 *   - the second page, 工程细节: prompts are read in chunks of up to 8,192
 *     tokens, and the expert products run on the quantised weights without
 *     first expanding them to FP16 in memory.
 *   - the second page, 代码结构: a router kernel and an MoE kernel on the GPU.
 *   The layer's specification fixes the rest: router logits l = W_r x (+ an
 *   optional per-expert bias), softmax over the experts, the k largest
 *   (ties to the lower expert index), their probabilities renormalised to
 *   sum to 1; each selected expert is a SwiGLU MLP on its 2-bit weights,
 *   h = silu(W_gate x) * (W_up x), o = W_down h; y = sum_j w_j o_j.
 *
 * Conventions
 *   - All tensor arguments are DEVICE pointers unless marked "host". The
 *     caller owns every tensor and stream; the library owns only the
 *     workspace it allocates when strata_moe_layer_create gets NULL.
 *   - Every compute call is asynchronous on `stream` and returns after
 *     enqueue. Argument errors are returned synchronously and nothing is
 *     enqueued. Device-side errors (a bounded wait that ran out) are recorded
 *     in a device status word read by strata_moe_check_status.
 *   - No C++ exception crosses this ABI. strata_last_error() gives a
 *     thread-local message for the last non-OK status of the calling thread.
 *   - Device pointers must be 16-byte aligned.
 *   - One layer handle serves one stream at a time: its workspace holds the
 *     routing of the last call.
 */
#ifndef STRATA_MOE_H
#define STRATA_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL means the legacy default stream. */
typedef struct CUstream_st *strata_stream_t;

typedef enum {
    STRATA_OK = 0,
    STRATA_ERR_INVALID_ARG = -1,    /* bad pointer, size, alignment or desc */
    STRATA_ERR_UNSUPPORTED = -2,    /* shape, format or flag the library does not run */
    STRATA_ERR_CUDA = -3,           /* a CUDA runtime call failed */
    STRATA_ERR_OOM = -4,            /* workspace allocation failed */
    STRATA_ERR_TOO_MANY_TOKENS = -5,/* n_tokens > max_tokens (layer calls) */
    STRATA_ERR_BAD_BLOB = -6,       /* blob pointer or packer input invalid */
    STRATA_ERR_TIMEOUT = -7,        /* a device wait exceeded its time limit */
    STRATA_ERR_BOUNDS = -8          /* checked build: an index taken from data was out of range */
} strata_status;

/* ------------------------------------------------------------------ format
 * STRATA_FMT_Q2_0_TILED: the 2-bit block format ("Q2_0" on the pages, first
 * page, 功能与原则; its bits are this library's).
 *   weight W[r][k] = (c[r][k] - 1.5) * s[r][k/32], c in {0,1,2,3}, s fp16:
 *   32-weight blocks along the reduction dimension K of each output row.
 * A matrix [R x K] (R % 64 == 0, K % 64 == 0) is stored as tiles, one per
 * (64-row panel p, 64-column slice s); a tile is 1280 bytes:
 *   bytes [0, 1024):   codes, row i (0..63) at bytes 16i..16i+15, as four
 *                      little-endian uint32 words W0..W3; column c (0..63)
 *                      of the tile, written c = 16j + 8s + 2t + h (j < 4,
 *                      s < 2, t < 4, h < 2), lives in word Wt at bit
 *                      16h + 8s + 6 - 2j. Word t thus holds exactly the 16
 *                      codes that lane t of a 4-lane group needs for the
 *                      row in the warp-level 16x8x16 MMA fragment layout
 *                      (columns 2t, 2t+1, 2t+8, 2t+9 of each 16-column
 *                      step), and one mask per register extracts the two
 *                      codes of a column pair without a shift;
 *   bytes [1024, 1280): scales, row i at 1024+4i: fp16 (little-endian) of
 *                      block 2s, then of block 2s+1.
 * Every tile is a multiple of 16 bytes, so tiles serve 128-bit loads and
 * 1-D bulk (TMA) copies alike. A lone matrix (strata_q2_pack) keeps its
 * tiles in (p, s) order: tile (p, s) at byte (p * K/64 + s) * 1280.
 *
 * Expert blob: experts 0..E-1 back to back, strata_moe_expert_bytes() each:
 *   gate/up section: for p in 0..f/64-1, for s in 0..d/64-1:
 *                    [gate tile (p,s)][up tile (p,s)]     (2560 bytes)
 *   down section:    down matrix [d x f], for s in 0..f/64-1 (its K slices),
 *                    for p in 0..d/64-1: tile (p,s)       (1280 bytes each)
 *   per expert: 3*d*f/32*10 bytes (d=2048, f=768: 1,474,560 bytes).
 * The order keeps, contiguous in memory, everything one 64-row slice of the
 * expert's hidden layer needs: its gate and up rows over all of K
 * ((d/64) * 2560 bytes) and the down columns it feeds ((d/64) * 1280
 * bytes); the tensor-core path's 128-row panels are two adjacent 64-row
 * tiles (down) or two 2560-byte pairs (gate/up).
 *
 * STRATA_FMT_Q4_0_TILED: the 4-bit block level. The pages' quality ladder
 * (first page, 能跑多快, its table: Q2_0, IQ2_XS, IQ3_XXS, IQ3_S) has wider
 * levels but does not print their bits; this one is the 2-bit rule with
 * 4-bit codes, this library's own:
 *   weight W[r][k] = (c[r][k] - 7.5) * s[r][k/32], c in {0..15}, s fp16.
 * The same 64 x 64 tiles, 2304 bytes each:
 *   bytes [0, 2048):   codes, row i at bytes 32i..32i+31, eight
 *                      little-endian uint32 words W0..W7; column
 *                      c = 16j + 8s + 2t + h lives in word W(2t + j/2) at
 *                      bits 16h + 8(j%2) + 4s .. +3. Lane t of a 4-lane
 *                      group reads W(2t), W(2t+1) (one 8-byte load) and
 *                      holds every code of its fragment columns; one mask
 *                      per register extracts a column pair;
 *   bytes [2048, 2304): scales, row i at 2048+4i, as in the 2-bit tile.
 * Expert blob and tile order as above with 2304-byte tiles: gate/up pairs of
 * 4608 bytes, 3*d*f/32*18 bytes per expert (d=2048, f=768: 2,654,208).
 */
#define STRATA_FMT_Q2_0_TILED 1
#define STRATA_FMT_Q4_0_TILED 2
#define STRATA_Q2_TILE_ROWS 64
#define STRATA_Q2_TILE_COLS 64
#define STRATA_Q2_TILE_BYTES 1280
#define STRATA_Q4_TILE_BYTES 2304

/* desc.flags */
#define STRATA_ACCUMULATE 1u      /* y += MoE(x) instead of y = MoE(x) */
#define STRATA_FORCE_PREFILL 2u   /* use the tensor-core path even for <= 16 tokens */

/* Largest token count served by the streaming (decode/verify) path. */
#define STRATA_DECODE_MAX_TOKENS 16

typedef struct {
    int32_t d_model;      /* d, multiple of 128 */
    int32_t d_ff;         /* f, expert intermediate size, multiple of 128 */
    int32_t n_experts;    /* E, 1..1024 */
    int32_t top_k;        /* k, 1 <= k <= min(E, 32) */
    int32_t max_tokens;   /* largest n_tokens of one layer call (workspace size) */
    int32_t block_size;   /* must be 32 */
    int32_t weight_format;/* STRATA_FMT_Q2_0_TILED or STRATA_FMT_Q4_0_TILED */
    uint32_t flags;       /* STRATA_ACCUMULATE | STRATA_FORCE_PREFILL */
    const float *router_bias; /* device fp32 [E] added to the logits, or NULL */
} strata_moe_desc;

typedef struct strata_moe_layer_s *strata_moe_layer;

/* Bytes of one packed matrix [rows x K] (rows % 64 == 0, K % 64 == 0), 2-bit
 * and 4-bit format; 0 for other shapes. */
size_t strata_q2_matrix_bytes(int32_t rows, int32_t K);
size_t strata_q4_matrix_bytes(int32_t rows, int32_t K);
/* Bytes of one packed expert: 3*d*f/32*10 (2-bit), 3*d*f/32*18 (4-bit). */
size_t strata_moe_expert_bytes(const strata_moe_desc *desc);
/* Bytes of the whole expert blob of a layer: E * strata_moe_expert_bytes. */
size_t strata_moe_expert_blob_bytes(const strata_moe_desc *desc);
/* Device workspace a layer handle needs for desc->max_tokens tokens. */
size_t strata_moe_workspace_bytes(const strata_moe_desc *desc);

/* Validate desc and build a layer handle. workspace: device memory of at
 * least strata_moe_workspace_bytes(desc) bytes owned by the caller, or NULL
 * to let the library allocate (and later free) it. The current CUDA device
 * at create time is the device every later call must run on.
 * Errors: INVALID_ARG / UNSUPPORTED (desc), OOM, CUDA. */
strata_status strata_moe_layer_create(const strata_moe_desc *desc, void *workspace,
                                      size_t workspace_bytes, strata_moe_layer *out);
/* Free the handle (and the workspace if the library allocated it). The
 * caller must make sure no work using it is still queued. */
strata_status strata_moe_layer_destroy(strata_moe_layer layer);

/* One MoE layer: y (=|+=) sum_j w_j * SwiGLU_{e_j}(x) for every token.
 *   x_bf16      [n_tokens x d] bf16, row-major
 *   router_w    [E x d] fp32, row-major (router bias: desc.router_bias)
 *   expert_blob E packed experts (format above)
 *   y           [n_tokens x d] fp32
 * n_tokens in 0..max_tokens (0 is a no-op). n_tokens <= 16 runs the whole
 * layer as one cooperative kernel that streams only the selected experts'
 * weights (warp-level MMA on codes decoded in registers); larger calls run
 * the tensor-core router, the routing kernels and the grouped tensor-core
 * expert GEMMs. Both multiply fp16 operands with fp32 accumulation; each
 * token's x is scaled by a power of two (its largest |x| to [1, 2)) before
 * the fp16 conversion and the results are scaled back exactly, so any bf16
 * magnitude keeps full precision. Errors: INVALID_ARG, TOO_MANY_TOKENS, CUDA. */
strata_status strata_moe_forward(strata_moe_layer layer, const void *x_bf16, const float *router_w,
                                 const void *expert_blob, float *y, int32_t n_tokens,
                                 strata_stream_t stream);

/* Router logits only (step one of the layer): logits [n_tokens x E] fp32 =
 * x W_r^T + bias. Same paths and precision as inside strata_moe_forward. */
strata_status strata_moe_router_logits(strata_moe_layer layer, const void *x_bf16,
                                       const float *router_w, float *logits, int32_t n_tokens,
                                       strata_stream_t stream);

/* Routing only: logits, softmax top-k, renormalised weights and the
 * per-expert token lists, kept in the workspace for strata_moe_experts and
 * strata_moe_get_routing. */
strata_status strata_moe_route(strata_moe_layer layer, const void *x_bf16, const float *router_w,
                               int32_t n_tokens, strata_stream_t stream);

/* Expert computation and combine for the routing of the last
 * strata_moe_route call on this handle (same x and n_tokens), or of the last
 * strata_moe_forward if that call took the tensor-core path (more than 16
 * tokens, or STRATA_FORCE_PREFILL). Errors: INVALID_ARG when the handle's last
 * routing call was not one of these, or had another n_tokens (a forward of
 * <= 16 tokens on the one-launch path and a stack keep no tile lists). */
strata_status strata_moe_experts(strata_moe_layer layer, const void *x_bf16, const void *expert_blob,
                                 float *y, int32_t n_tokens, strata_stream_t stream);

/* Copy the routing of the last call into caller buffers (device pointers;
 * any may be NULL):
 *   topk_idx [T x k] int32, experts of each token in rank order
 *            (logit descending, ties to the lower index)
 *   topk_w   [T x k] fp32, renormalised softmax weights
 *   expert_offsets [E + 1] int32, start of each expert's list
 *   token_list [T*k] int32, tokens of each expert in ascending order
 *   pair_slot  [T*k] int32, slot j at which the token chose that expert */
strata_status strata_moe_get_routing(strata_moe_layer layer, int32_t *topk_idx, float *topk_w,
                                     int32_t *expert_offsets, int32_t *token_list,
                                     int32_t *pair_slot, strata_stream_t stream);

/* Routing without any allocation, for callers that cannot allocate device
 * memory when they route (all free memory handed to another allocator, or a
 * loop that must not call cudaMalloc / cudaFree because they can synchronise
 * the device). The pages have no counterpart of this call: it is this
 * library's own interface.
 *
 * Computes what strata_moe_route computes for desc (router bias from
 * desc->router_bias; max_tokens and flags are not used and not checked) and
 * writes it to the
 * caller's device buffers, laid out as strata_moe_get_routing documents:
 * topk_idx [T x k], topk_w [T x k], expert_offsets [E + 1],
 * token_list [T*k], pair_slot [T*k] (all required, 4-byte aligned).
 * x_bf16 [T x d] and router_w [E x d] as for strata_moe_route (16-byte
 * aligned).
 *
 * Limit: n_tokens <= STRATA_NOALLOC_MAX_TOKENS (16); larger counts return
 * STRATA_ERR_TOO_MANY_TOKENS. The kernels' scratch is a fixed array of
 * STRATA_NOALLOC_SCRATCH_BYTES in device memory owned by the library, one per
 * device, whose address is looked up by the first call on each device, and
 * again after the device's context changes (a cudaDeviceReset); make that
 * first call before capturing a stream that contains the call. No scratch
 * word needs to start at zero. Calls on one device share that array:
 * calls whose device work may overlap race on it, so issue them in order
 * (e.g. on one stream). Asynchronous on `stream`. */
#define STRATA_NOALLOC_MAX_TOKENS 16
#define STRATA_NOALLOC_SCRATCH_BYTES (112 * 1024)
strata_status strata_moe_route_noalloc(const strata_moe_desc *desc, const void *x_bf16,
                                       const float *router_w, int32_t n_tokens, int32_t *topk_idx,
                                       float *topk_w, int32_t *expert_offsets, int32_t *token_list,
                                       int32_t *pair_slot, strata_stream_t stream);

/* A stack of n_layers layers with the residual recurrence
 *   x <- x + MoE_l(bf16(RMSNorm(x)))   (RMSNorm with unit weights, eps)
 * x_resid [n_tokens x d] fp32 in/out. router_w, router_bias and
 * expert_blobs are HOST arrays of n_layers device pointers (router_bias may
 * be NULL, or hold NULL entries). n_tokens may exceed max_tokens: tokens are
 * processed in chunks of max_tokens, each chunk through all layers. The
 * decode-size sequence is captured into a CUDA graph on first use and
 * replayed while the pointers stay the same (not when the stream is already
 * capturing). desc.flags STRATA_ACCUMULATE is ignored here. */
strata_status strata_moe_stack_forward(strata_moe_layer layer, int32_t n_layers,
                                       const float *const *router_w,
                                       const float *const *router_bias,
                                       const void *const *expert_blobs, float *x_resid,
                                       int32_t n_tokens, float rms_eps, strata_stream_t stream);

/* RMSNorm with unit weights, rounded to bf16 (step of the stack):
 * out[t][i] = bf16_rne(x[t][i] / sqrt(mean_i x[t][i]^2 + eps)). */
strata_status strata_rmsnorm_bf16(const float *x, void *out_bf16, int32_t n_tokens, int32_t d,
                                  float eps, strata_stream_t stream);

/* Stage timing hook. events: HOST array of n_events cudaEvent_t handles
 * created by the caller. With n_events == 5, every later forward / experts
 * call on this handle records, on its stream: events[0] at its start,
 * [1] after routing, [2] right before and [3] right after the dominant
 * kernel (decode: the one-launch layer kernel, so [1] coincides with [0];
 * prefill: the gate/up tensor-core GEMM), [4] at its end. n_events == 0
 * removes the hook.
 * Errors: INVALID_ARG for any other count. */
strata_status strata_moe_set_stage_events(strata_moe_layer layer, void *const *events, int32_t n_events);

/* Synchronise the layer's stream work and read its device status word
 * (OK, TIMEOUT if a bounded device wait ran out, BOUNDS if a check of the
 * checked build failed); clears the word. */
strata_status strata_moe_check_status(strata_moe_layer layer);

/* Pack one matrix on the HOST: codes [rows x K] one code (0..3) per byte,
 * scales [rows x K/32] fp16 bits, into dst (host, strata_q2_matrix_bytes).
 * Errors: BAD_BLOB (a code > 3), INVALID_ARG. */
strata_status strata_q2_pack(const uint8_t *codes, const uint16_t *scales_fp16, int32_t rows,
                             int32_t K, void *dst);
/* The same for the 4-bit format: codes 0..15, dst strata_q4_matrix_bytes.
 * Errors: BAD_BLOB (a code > 15), INVALID_ARG. */
strata_status strata_q4_pack(const uint8_t *codes, const uint16_t *scales_fp16, int32_t rows,
                             int32_t K, void *dst);

/* Pack one expert on the HOST into its blob section (dst: host,
 * strata_moe_expert_bytes) in desc->weight_format: gate/up [f x d], down
 * [d x f], one code per byte (0..3 or 0..15). Errors: BAD_BLOB (a code out
 * of range), INVALID_ARG, UNSUPPORTED (desc). */
strata_status strata_moe_pack_expert(const strata_moe_desc *desc, const uint8_t *gate_codes,
                                     const uint16_t *gate_scales, const uint8_t *up_codes,
                                     const uint16_t *up_scales, const uint8_t *down_codes,
                                     const uint16_t *down_scales, void *dst);

/* Same as strata_moe_pack_expert with device pointers, on `stream`. Codes
 * above the format's largest (3 or 15) are masked to its 2 or 4 bits. */
strata_status strata_moe_pack_expert_device(const strata_moe_desc *desc, const uint8_t *gate_codes,
                                            const uint16_t *gate_scales, const uint8_t *up_codes,
                                            const uint16_t *up_scales, const uint8_t *down_codes,
                                            const uint16_t *down_scales, void *dst,
                                            strata_stream_t stream);

/* Checked build. The library compiled with -DSTRATA_CHECKED
 * (libstrata_moe_checked.so) tests every index its kernels take from data
 * (selected experts, tokens of the per-expert lists, list positions, pair
 * slots, GEMM tile entries) before using it; a bad index is recorded in the
 * device status word and the access skipped or redirected to a harmless one,
 * so a corrupted routing shows up as STRATA_ERR_BOUNDS from
 * strata_moe_check_status instead of a fault. The normal build compiles the
 * checks away. Same API and results otherwise.
 * strata_is_checked_build: 1 for the checked build, 0 otherwise.
 * strata_selftest_bounds_check: launches a kernel that tests an index one
 * past the end of an array (and skips that access); synchronous. Returns
 * STRATA_ERR_BOUNDS in the checked build, STRATA_OK in the normal one. */
int32_t strata_is_checked_build(void);
strata_status strata_selftest_bounds_check(strata_stream_t stream);

/* Failure-detection self test: launches a kernel whose bounded wait polls a
 * flag that nothing sets, for timeout_ns nanoseconds (1e3..1e10), then
 * returns; reports STRATA_ERR_TIMEOUT through the status word like any
 * other wait. Synchronous. */
strata_status strata_selftest_wait_timeout(uint64_t timeout_ns, strata_stream_t stream);

const char *strata_status_string(strata_status s);
const char *strata_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* STRATA_MOE_H */
