// strata_moe.cu -- host side of the C ABI (include/strata_moe.h): argument
// validation, workspace planning, tensor-map set-up, launch sequencing of
// the decode (streaming) and prefill (tensor-core) paths, the layer stack
// with CUDA-graph replay, the packers and status reporting.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>
#include <vector>

#include "../../include/strata_moe.h"
#include "abi_internal.h"
#include "common.cuh"
#include "kernels.h"

using namespace strata;

// ------------------------------------------------------------ errors
static thread_local char g_last_error[512] = "";

static strata_status fail(strata_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return s;
}

#define CUDA_TRY(expr)                                                                                  \
    do {                                                                                                \
        cudaError_t e_ = (expr);                                                                        \
        if (e_ != cudaSuccess) return fail(STRATA_ERR_CUDA, "%s: %s", #expr, cudaGetErrorString(e_)); \
    } while (0)

static strata_status check_launch(const char *what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(STRATA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return STRATA_OK;
}

extern "C" const char *strata_status_string(strata_status s) {
    switch (s) {
        case STRATA_OK: return "ok";
        case STRATA_ERR_INVALID_ARG: return "invalid argument";
        case STRATA_ERR_UNSUPPORTED: return "unsupported";
        case STRATA_ERR_CUDA: return "CUDA error";
        case STRATA_ERR_OOM: return "out of memory";
        case STRATA_ERR_TOO_MANY_TOKENS: return "too many tokens";
        case STRATA_ERR_BAD_BLOB: return "bad expert blob";
        case STRATA_ERR_TIMEOUT: return "device wait timed out";
        case STRATA_ERR_BOUNDS: return "bounds check failed";
    }
    return "unknown status";
}

extern "C" const char *strata_last_error(void) { return g_last_error; }

// ------------------------------------------------------------ sizes
namespace strata {
size_t expert_bytes(const Shape &s) { return (size_t)3 * (s.d / 64) * (s.f / 64) * tile_bytes(s); }
size_t down_section_offset(const Shape &s) { return (size_t)2 * (s.d / 64) * (s.f / 64) * tile_bytes(s); }
}  // namespace strata

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static strata_status validate_desc(const strata_moe_desc *d) {
    if (!d) return fail(STRATA_ERR_INVALID_ARG, "desc is NULL");
    if (d->block_size != 32) return fail(STRATA_ERR_UNSUPPORTED, "block_size must be 32 (got %d)", d->block_size);
    if (d->weight_format != STRATA_FMT_Q2_0_TILED && d->weight_format != STRATA_FMT_Q4_0_TILED)
        return fail(STRATA_ERR_UNSUPPORTED, "weight_format must be STRATA_FMT_Q2_0_TILED or STRATA_FMT_Q4_0_TILED");
    if (d->d_model <= 0 || d->d_model % 128 || d->d_model > 16384)
        return fail(STRATA_ERR_INVALID_ARG, "d_model must be a positive multiple of 128 <= 16384 (got %d)",
                    d->d_model);
    if (d->d_ff <= 0 || d->d_ff % 128 || d->d_ff > 16384)
        return fail(STRATA_ERR_INVALID_ARG, "d_ff must be a positive multiple of 128 <= 16384 (got %d)", d->d_ff);
    if (d->n_experts < 1 || d->n_experts > 1024)
        return fail(STRATA_ERR_INVALID_ARG, "n_experts must be in 1..1024 (got %d)", d->n_experts);
    if (d->top_k < 1 || d->top_k > 32 || d->top_k > d->n_experts)
        return fail(STRATA_ERR_INVALID_ARG, "top_k must be in 1..min(n_experts, 32) (got %d)", d->top_k);
    if (d->max_tokens < 1 || d->max_tokens > 65536)
        return fail(STRATA_ERR_INVALID_ARG, "max_tokens must be in 1..65536 (got %d)", d->max_tokens);
    if (d->flags & ~(STRATA_ACCUMULATE | STRATA_FORCE_PREFILL))
        return fail(STRATA_ERR_INVALID_ARG, "unknown flag bits 0x%x", d->flags);
    if (d->router_bias && !aligned16(d->router_bias))
        return fail(STRATA_ERR_INVALID_ARG, "router_bias must be 16-byte aligned");
    return STRATA_OK;
}

strata_status strata_set_error(strata_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return s;
}

strata_status strata_check_desc(const strata_moe_desc *desc) { return validate_desc(desc); }

static Shape shape_of(const strata_moe_desc *d) {
    return Shape{d->d_model, d->d_ff, d->n_experts, d->top_k, d->weight_format == STRATA_FMT_Q4_0_TILED ? 4 : 2};
}

// Workspace plan: offsets of every buffer in one allocation (256-B aligned).
struct Plan {
    size_t off[24];
    size_t total;
    int max_tiles1, max_tiles2;
};

static Plan plan_workspace(const strata_moe_desc *d) {
    const Shape s = shape_of(d);
    const size_t T = (size_t)d->max_tokens, k = s.k, E = s.E;
    const size_t P = T * k;
    const size_t nblk = (T + kRouteBlock - 1) / kRouteBlock;
    Plan p{};
    p.max_tiles1 = (int)((P + kGemm1N - 1) / kGemm1N + E);
    p.max_tiles2 = (int)((P + kGemm2N - 1) / kGemm2N + E);
    const size_t sz[24] = {
        256,                                      // 0 status
        64 * 4,                                   // 1 meta
        T * E * 4,                                // 2 logits
        P * 4,                                    // 3 topk_idx
        P * 4,                                    // 4 topk_w
        E * 4,                                    // 5 counts
        (E + 1) * 4,                              // 6 offsets
        P * 4,                                    // 7 token_list
        P * 4,                                    // 8 pair_slot
        P * 4,                                    // 9 pair_w
        P * 4,                                    // 10 pair_of
        nblk * E * 4,                             // 11 blk_counts
        E * 4,                                    // 12 act
        (size_t)kDecMaxT * E * 4 * 4,             // 13 lpart
        P * (size_t)s.d * 2,                      // 14 xp
        P * (size_t)s.f * 2,                      // 15 hbuf
        (size_t)p.max_tiles1 * 16,                // 16 tiles1
        (size_t)p.max_tiles2 * 16,                // 17 tiles2
        T * (size_t)s.d * 2,                      // 18 xn
        (2 + E) * 4,                              // 19 sync
        E * (size_t)s.d * 2,                      // 20 w_hi
        E * (size_t)s.d * 2,                      // 21 w_lo
        P * 4,                                    // 22 pair_s
        T * 4,                                    // 23 tok_s
    };
    size_t o = 0;
    for (int i = 0; i < 24; ++i) {
        p.off[i] = o;
        o += (sz[i] + 255) & ~(size_t)255;
    }
    p.total = o;
    return p;
}

static Workspace carve(uint8_t *base, const Plan &p) {
    Workspace w;
    w.status = reinterpret_cast<uint32_t *>(base + p.off[0]);
    w.meta = reinterpret_cast<int32_t *>(base + p.off[1]);
    w.logits = reinterpret_cast<float *>(base + p.off[2]);
    w.topk_idx = reinterpret_cast<int32_t *>(base + p.off[3]);
    w.topk_w = reinterpret_cast<float *>(base + p.off[4]);
    w.counts = reinterpret_cast<int32_t *>(base + p.off[5]);
    w.offsets = reinterpret_cast<int32_t *>(base + p.off[6]);
    w.token_list = reinterpret_cast<int32_t *>(base + p.off[7]);
    w.pair_slot = reinterpret_cast<int32_t *>(base + p.off[8]);
    w.pair_w = reinterpret_cast<float *>(base + p.off[9]);
    w.pair_of = reinterpret_cast<int32_t *>(base + p.off[10]);
    w.blk_counts = reinterpret_cast<int32_t *>(base + p.off[11]);
    w.act = reinterpret_cast<int32_t *>(base + p.off[12]);
    w.lpart = reinterpret_cast<float *>(base + p.off[13]);
    w.xp = base + p.off[14];
    w.hbuf = base + p.off[15];
    w.tiles1 = reinterpret_cast<int4 *>(base + p.off[16]);
    w.tiles2 = reinterpret_cast<int4 *>(base + p.off[17]);
    w.xn = base + p.off[18];
    w.sync = reinterpret_cast<uint32_t *>(base + p.off[19]);
    w.w_hi = base + p.off[20];
    w.w_lo = base + p.off[21];
    w.pair_s = reinterpret_cast<float *>(base + p.off[22]);
    w.tok_s = reinterpret_cast<float *>(base + p.off[23]);
    return w;
}

// ------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// Maps over a row-major fp16 matrix [rows x K]: boxes of 64 columns x
// (16, 32, 64, 128, 256) rows, 128-byte swizzle (the operand layout of the
// tensor-core kernels).
static strata_status make_maps(TmaMaps &m, void *base, size_t rows, int K) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return fail(STRATA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    for (int i = 0; i < 5; ++i) {
        cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
        cuuint64_t strides[1] = {(cuuint64_t)K * 2};
        cuuint32_t box[2] = {64, (cuuint32_t)(16 << i)};
        cuuint32_t es[2] = {1, 1};
        CUresult r = enc(&m.m[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, base, dims, strides, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return fail(STRATA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    }
    return STRATA_OK;
}

// Map over a row-major bf16 matrix [rows x K] with boxes of 64 columns x
// box_rows rows and 128-byte swizzle; rows beyond the matrix read as zeros.
static strata_status make_bf16_map(CUtensorMap *m, const void *base, size_t rows, int K, int box_rows) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return fail(STRATA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(STRATA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return STRATA_OK;
}

namespace strata {
cudaError_t init_gemm_attributes(int max_smem);
static cudaError_t init_kernel_attributes(int device, const Shape &s, int max_tokens, int num_sms) {
    int max_smem = 0;
    cudaError_t e = cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
    if (e == cudaSuccess) e = init_gemm_attributes(max_smem);
    if (e == cudaSuccess) e = init_router_attributes(max_smem);
    if (e == cudaSuccess) e = init_fused_attributes(s, max_tokens, max_smem, num_sms);
    return e;
}
}  // namespace strata

// ------------------------------------------------------------ layer
struct StackGraph {
    cudaGraphExec_t exec = nullptr;
    std::vector<const void *> key;
};

struct strata_moe_layer_s {
    strata_moe_desc desc;
    cudaStream_t capture_stream;  // private stream the stack graph is captured on
    Shape shape;
    int device;
    int num_sms;
    void *ws_mem;
    bool owns_ws;
    Plan plan;
    Workspace ws;
    TmaMaps maps1, maps2;
    RouterMaps rmaps;  // W_hi / W_lo fixed at creation; x encoded per call
    bool fused_ok;   // the one-launch streaming layer fits this shape
    int max_smem;
    StackGraph graph;
    cudaEvent_t stage_ev[5];
    bool stage_on;
    // n_tokens of the last call whose routing built the expert GEMMs' tile
    // lists (strata_moe_route, or a forward on the tensor-core path); -1 after
    // a call that did not (the one-launch decode layer, a stack)
    int tiled_tokens;
};

static void stage_mark(strata_moe_layer L, int i, cudaStream_t st) {
    if (L->stage_on) cudaEventRecordWithFlags(L->stage_ev[i], st, cudaEventRecordExternal);
}

extern "C" strata_status strata_moe_set_stage_events(strata_moe_layer L, void *const *events, int32_t n) {
    if (!L) return fail(STRATA_ERR_INVALID_ARG, "layer is NULL");
    if (n == 0) {
        L->stage_on = false;
        return STRATA_OK;
    }
    if (n != 5 || !events) return fail(STRATA_ERR_INVALID_ARG, "stage events: need 5 events (got %d)", n);
    for (int i = 0; i < 5; ++i) {
        if (!events[i]) return fail(STRATA_ERR_INVALID_ARG, "stage event %d is NULL", i);
        L->stage_ev[i] = static_cast<cudaEvent_t>(events[i]);
    }
    L->stage_on = true;
    return STRATA_OK;
}

extern "C" size_t strata_q2_matrix_bytes(int32_t rows, int32_t K) {
    if (rows <= 0 || K <= 0 || rows % STRATA_Q2_TILE_ROWS || K % STRATA_Q2_TILE_COLS) return 0;
    return (size_t)(rows / 64) * (K / 64) * STRATA_Q2_TILE_BYTES;
}

extern "C" size_t strata_q4_matrix_bytes(int32_t rows, int32_t K) {
    if (rows <= 0 || K <= 0 || rows % STRATA_Q2_TILE_ROWS || K % STRATA_Q2_TILE_COLS) return 0;
    return (size_t)(rows / 64) * (K / 64) * STRATA_Q4_TILE_BYTES;
}

extern "C" size_t strata_moe_expert_bytes(const strata_moe_desc *desc) {
    if (validate_desc(desc) != STRATA_OK) return 0;
    return expert_bytes(shape_of(desc));
}

extern "C" size_t strata_moe_expert_blob_bytes(const strata_moe_desc *desc) {
    if (validate_desc(desc) != STRATA_OK) return 0;
    return expert_bytes(shape_of(desc)) * (size_t)desc->n_experts;
}

extern "C" size_t strata_moe_workspace_bytes(const strata_moe_desc *desc) {
    if (validate_desc(desc) != STRATA_OK) return 0;
    return plan_workspace(desc).total;
}

extern "C" strata_status strata_moe_layer_create(const strata_moe_desc *desc, void *workspace, size_t workspace_bytes,
                                                 strata_moe_layer *out) {
    if (!out) return fail(STRATA_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    strata_status s = validate_desc(desc);
    if (s != STRATA_OK) return s;
    Plan plan = plan_workspace(desc);
    if (workspace) {
        if (workspace_bytes < plan.total)
            return fail(STRATA_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", workspace_bytes, plan.total);
        if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
            return fail(STRATA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    }
    auto *L = new (std::nothrow) strata_moe_layer_s();
    if (!L) return fail(STRATA_ERR_OOM, "host allocation failed");
    L->desc = *desc;
    L->shape = shape_of(desc);
    L->plan = plan;
    L->tiled_tokens = -1;
    if (cudaGetDevice(&L->device) != cudaSuccess ||
        cudaDeviceGetAttribute(&L->num_sms, cudaDevAttrMultiProcessorCount, L->device) != cudaSuccess) {
        delete L;
        return fail(STRATA_ERR_CUDA, "no CUDA device");
    }
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, L->device);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, L->device);
    if (major != 10 || minor != 0) {
        delete L;
        return fail(STRATA_ERR_UNSUPPORTED, "this library is built for sm_100a (B200); device is sm_%d%d", major,
                    minor);
    }
    if (workspace) {
        L->ws_mem = workspace;
        L->owns_ws = false;
    } else {
        if (cudaMalloc(&L->ws_mem, plan.total) != cudaSuccess) {
            cudaGetLastError();
            delete L;
            return fail(STRATA_ERR_OOM, "cudaMalloc of %zu workspace bytes failed", plan.total);
        }
        L->owns_ws = true;
    }
    L->ws = carve(static_cast<uint8_t *>(L->ws_mem), plan);
    if (cudaMemset(L->ws_mem, 0, plan.off[2]) != cudaSuccess) {  // status + meta
        if (L->owns_ws) cudaFree(L->ws_mem);
        delete L;
        return fail(STRATA_ERR_CUDA, "workspace clear failed");
    }
    const size_t P = (size_t)desc->max_tokens * desc->top_k;
    if ((s = make_maps(L->maps1, L->ws.xp, P, L->shape.d)) != STRATA_OK ||
        (s = make_maps(L->maps2, L->ws.hbuf, P, L->shape.f)) != STRATA_OK ||
        (s = make_bf16_map(&L->rmaps.w_hi, L->ws.w_hi, L->shape.E, L->shape.d, 128)) != STRATA_OK ||
        (s = make_bf16_map(&L->rmaps.w_lo, L->ws.w_lo, L->shape.E, L->shape.d, 128)) != STRATA_OK) {
        if (L->owns_ws) cudaFree(L->ws_mem);
        delete L;
        return s;
    }
    {
        int max_smem = 0;
        cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, L->device);
        const int Tw = desc->max_tokens < kDecMaxT ? desc->max_tokens : kDecMaxT;
        L->fused_ok = decode_fused_supported(L->shape, Tw, max_smem, L->num_sms);
        L->max_smem = max_smem;
    }
    if (cudaMemset(L->ws.sync, 0, (size_t)(2 + L->shape.E) * 4) != cudaSuccess) {
        if (L->owns_ws) cudaFree(L->ws_mem);
        delete L;
        return fail(STRATA_ERR_CUDA, "workspace clear failed");
    }
    if (cudaError_t e = init_kernel_attributes(L->device, L->shape, desc->max_tokens, L->num_sms)) {
        cudaGetLastError();
        if (L->owns_ws) cudaFree(L->ws_mem);
        delete L;
        return fail(STRATA_ERR_CUDA, "kernel attribute set-up failed: %s", cudaGetErrorString(e));
    }
    *out = L;
    return STRATA_OK;
}

extern "C" strata_status strata_moe_layer_destroy(strata_moe_layer L) {
    if (!L) return STRATA_OK;
    if (L->graph.exec) cudaGraphExecDestroy(L->graph.exec);
    if (L->capture_stream) cudaStreamDestroy(L->capture_stream);
    if (L->owns_ws) cudaFree(L->ws_mem);
    delete L;
    return STRATA_OK;
}

static strata_status check_layer(strata_moe_layer L, int32_t T, bool layer_call) {
    if (!L) return fail(STRATA_ERR_INVALID_ARG, "layer is NULL");
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != L->device)
        return fail(STRATA_ERR_INVALID_ARG, "current device %d is not the layer's device %d", dev, L->device);
    if (T < 0) return fail(STRATA_ERR_INVALID_ARG, "n_tokens < 0");
    if (layer_call && T > L->desc.max_tokens)
        return fail(STRATA_ERR_TOO_MANY_TOKENS, "n_tokens %d > max_tokens %d", T, L->desc.max_tokens);
    return STRATA_OK;
}

static bool use_decode(strata_moe_layer L, int T) {
    return T <= kDecMaxT && L->fused_ok && !(L->desc.flags & STRATA_FORCE_PREFILL);
}

// logits of T tokens: GEMV for decode sizes, the tensor-core GEMM (bf16
// split of W) beyond
static strata_status router_impl(strata_moe_layer L, const void *x, const float *W, const float *bias, float *logits,
                                 int T, cudaStream_t st) {
    if (T <= kDecMaxT) {
        launch_router_gemv(x, W, bias, logits, T, L->shape, st);
        return STRATA_OK;
    }
    RouterMaps maps = L->rmaps;
    strata_status s = make_bf16_map(&maps.x, x, (size_t)T, L->shape.d, 256);
    if (s != STRATA_OK) return s;
    launch_router_tc(L->ws, maps, W, bias, logits, T, L->shape, L->num_sms, st);
    return STRATA_OK;
}

static strata_status route_impl(strata_moe_layer L, const void *x, const float *W, const float *bias, int T,
                                cudaStream_t st) {
    strata_status s = router_impl(L, x, W, bias, L->ws.logits, T, st);
    if (s != STRATA_OK) return s;
    launch_route_large(L->ws, T, L->plan.max_tiles1, L->plan.max_tiles2, L->shape, st, x);
    L->tiled_tokens = T;
    return check_launch("routing kernels");
}

static strata_status experts_impl(strata_moe_layer L, const void *x, const void *blob, float *y, int T, bool acc,
                                  cudaStream_t st) {
    const uint8_t *b = static_cast<const uint8_t *>(blob);
    launch_gather_xp(L->ws, x, T, L->shape, st);
    stage_mark(L, 2, st);
    launch_expert_gemm1(L->ws, b, L->maps1, L->plan.max_tiles1, T, L->shape, L->num_sms, st);
    stage_mark(L, 3, st);
    launch_expert_gemm2(L->ws, b, y, L->maps2, L->plan.max_tiles2, T, L->shape, L->num_sms, st);
    launch_combine(L->ws, y, acc, T, L->shape, st);  // y = (or +=) the sum of each token's k expert outputs
    return check_launch("expert kernels");
}

static strata_status check_io(const void *x, const float *W, const void *blob, const float *y) {
    if (!x || !W || !blob || !y) return fail(STRATA_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned16(x) || !aligned16(W) || !aligned16(y)) return fail(STRATA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    if (!aligned16(blob)) return fail(STRATA_ERR_BAD_BLOB, "expert blob must be 16-byte aligned");
    return STRATA_OK;
}

extern "C" strata_status strata_moe_forward(strata_moe_layer L, const void *x, const float *W, const void *blob,
                                            float *y, int32_t T, strata_stream_t stream) {
    strata_status s = check_layer(L, T, true);
    if (s != STRATA_OK) return s;
    if ((s = check_io(x, W, blob, y)) != STRATA_OK) return s;
    if (T == 0) return STRATA_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    stage_mark(L, 0, st);
    if (use_decode(L, T)) {
        L->tiled_tokens = -1;
        stage_mark(L, 1, st);
        cudaError_t e = launch_decode_fused(L->ws, x, W, L->desc.router_bias, static_cast<const uint8_t *>(blob), y,
                                            (L->desc.flags & STRATA_ACCUMULATE) != 0, false, 0.f, T, L->shape,
                                            L->num_sms, L->max_smem, st, L->stage_on ? L->stage_ev : nullptr);
        stage_mark(L, 4, st);
        if (e != cudaSuccess) return fail(STRATA_ERR_CUDA, "fused decode launch: %s", cudaGetErrorString(e));
        return check_launch("fused decode kernel");
    }
    if ((s = route_impl(L, x, W, L->desc.router_bias, T, st)) != STRATA_OK) return s;
    stage_mark(L, 1, st);
    s = experts_impl(L, x, blob, y, T, (L->desc.flags & STRATA_ACCUMULATE) != 0, st);
    stage_mark(L, 4, st);
    return s;
}

extern "C" strata_status strata_moe_router_logits(strata_moe_layer L, const void *x, const float *W, float *logits,
                                                  int32_t T, strata_stream_t stream) {
    strata_status s = check_layer(L, T, true);
    if (s != STRATA_OK) return s;
    if (!x || !W || !logits) return fail(STRATA_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned16(x) || !aligned16(W) || !aligned16(logits))
        return fail(STRATA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    if (T == 0) return STRATA_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if ((s = router_impl(L, x, W, L->desc.router_bias, logits, T, st)) != STRATA_OK) return s;
    return check_launch("router kernel");
}

extern "C" strata_status strata_moe_route(strata_moe_layer L, const void *x, const float *W, int32_t T,
                                          strata_stream_t stream) {
    strata_status s = check_layer(L, T, true);
    if (s != STRATA_OK) return s;
    if (!x || !W) return fail(STRATA_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned16(x) || !aligned16(W)) return fail(STRATA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    if (T == 0) return STRATA_OK;
    return route_impl(L, x, W, L->desc.router_bias, T, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" strata_status strata_moe_experts(strata_moe_layer L, const void *x, const void *blob, float *y, int32_t T,
                                            strata_stream_t stream) {
    strata_status s = check_layer(L, T, true);
    if (s != STRATA_OK) return s;
    if (!x || !blob || !y) return fail(STRATA_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned16(x) || !aligned16(y)) return fail(STRATA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    if (!aligned16(blob)) return fail(STRATA_ERR_BAD_BLOB, "expert blob must be 16-byte aligned");
    if (T == 0) return STRATA_OK;
    if (L->tiled_tokens != T)
        return fail(STRATA_ERR_INVALID_ARG,
                    "strata_moe_experts needs the routing of a strata_moe_route call with n_tokens = %d on this handle "
                    "(a forward of <= 16 tokens or a stack leaves none)", T);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    stage_mark(L, 1, st);
    s = experts_impl(L, x, blob, y, T, (L->desc.flags & STRATA_ACCUMULATE) != 0, st);
    stage_mark(L, 4, st);
    return s;
}

extern "C" strata_status strata_moe_get_routing(strata_moe_layer L, int32_t *topk_idx, float *topk_w,
                                                int32_t *expert_offsets, int32_t *token_list, int32_t *pair_slot,
                                                strata_stream_t stream) {
    strata_status s = check_layer(L, 0, false);
    if (s != STRATA_OK) return s;
    // the routing kernels record the token count of the last call in meta
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int32_t T = 0;
    CUDA_TRY(cudaMemcpyAsync(&T, L->ws.meta + META_N_TOKENS, sizeof T, cudaMemcpyDeviceToHost, st));
    CUDA_TRY(cudaStreamSynchronize(st));
    const size_t P = (size_t)T * L->shape.k;
    if (topk_idx) CUDA_TRY(cudaMemcpyAsync(topk_idx, L->ws.topk_idx, P * 4, cudaMemcpyDeviceToDevice, st));
    if (topk_w) CUDA_TRY(cudaMemcpyAsync(topk_w, L->ws.topk_w, P * 4, cudaMemcpyDeviceToDevice, st));
    if (expert_offsets)
        CUDA_TRY(cudaMemcpyAsync(expert_offsets, L->ws.offsets, (L->shape.E + 1) * 4, cudaMemcpyDeviceToDevice, st));
    if (token_list) CUDA_TRY(cudaMemcpyAsync(token_list, L->ws.token_list, P * 4, cudaMemcpyDeviceToDevice, st));
    if (pair_slot) CUDA_TRY(cudaMemcpyAsync(pair_slot, L->ws.pair_slot, P * 4, cudaMemcpyDeviceToDevice, st));
    return STRATA_OK;
}

extern "C" strata_status strata_rmsnorm_bf16(const float *x, void *out, int32_t T, int32_t d, float eps,
                                             strata_stream_t stream) {
    if (!x || !out) return fail(STRATA_ERR_INVALID_ARG, "NULL tensor pointer");
    if (T < 0 || d <= 0 || d % 8) return fail(STRATA_ERR_INVALID_ARG, "bad shape T=%d d=%d", T, d);
    if (!(eps >= 0.f)) return fail(STRATA_ERR_INVALID_ARG, "eps must be >= 0");
    launch_rmsnorm_bf16(x, out, T, d, eps, reinterpret_cast<cudaStream_t>(stream));
    return check_launch("rmsnorm kernel");
}

// One pass of the stack over tokens [t0, t0 + T).
static strata_status stack_enqueue(strata_moe_layer L, int n_layers, const float *const *W,
                                   const float *const *bias, const void *const *blobs, float *x, int T, float eps,
                                   cudaStream_t st) {
    strata_status s;
    if (use_decode(L, T)) {  // RMSNorm, routing and experts in one launch per layer
        for (int l = 0; l < n_layers; ++l) {
            const float *b = bias ? bias[l] : nullptr;
            cudaError_t e = launch_decode_fused(L->ws, x, W[l], b, static_cast<const uint8_t *>(blobs[l]), x, true,
                                                true, eps, T, L->shape, L->num_sms, L->max_smem, st, nullptr);
            if (e != cudaSuccess) return fail(STRATA_ERR_CUDA, "fused decode launch: %s", cudaGetErrorString(e));
        }
        return check_launch("fused decode kernels");
    }
    for (int l = 0; l < n_layers; ++l) {
        launch_rmsnorm_bf16(x, L->ws.xn, T, L->shape.d, eps, st);
        const float *b = bias ? bias[l] : nullptr;
        if ((s = route_impl(L, L->ws.xn, W[l], b, T, st)) != STRATA_OK) return s;
        if ((s = experts_impl(L, L->ws.xn, blobs[l], x, T, true, st)) != STRATA_OK) return s;
    }
    return STRATA_OK;
}

extern "C" strata_status strata_moe_stack_forward(strata_moe_layer L, int32_t n_layers, const float *const *W,
                                                  const float *const *bias, const void *const *blobs, float *x,
                                                  int32_t T, float eps, strata_stream_t stream) {
    strata_status s = check_layer(L, T, false);
    if (s != STRATA_OK) return s;
    if (n_layers < 0 || !W || !blobs || !x) return fail(STRATA_ERR_INVALID_ARG, "bad stack arguments");
    if (!(eps >= 0.f)) return fail(STRATA_ERR_INVALID_ARG, "eps must be >= 0");
    for (int l = 0; l < n_layers; ++l) {
        if (!W[l] || !blobs[l]) return fail(STRATA_ERR_INVALID_ARG, "NULL pointer for layer %d", l);
        if (!aligned16(W[l]) || !aligned16(blobs[l])) return fail(STRATA_ERR_INVALID_ARG, "layer %d pointers not 16-byte aligned", l);
        if (bias && bias[l] && !aligned16(bias[l])) return fail(STRATA_ERR_INVALID_ARG, "layer %d bias not aligned", l);
    }
    if (!aligned16(x)) return fail(STRATA_ERR_INVALID_ARG, "x_resid must be 16-byte aligned");
    if (T == 0 || n_layers == 0) return STRATA_OK;
    L->tiled_tokens = -1;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int chunk = L->desc.max_tokens;
    const bool decode = T <= chunk && use_decode(L, T);
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    CUDA_TRY(cudaStreamIsCapturing(st, &cap));
    if (!decode || cap != cudaStreamCaptureStatusNone) {
        for (int t0 = 0; t0 < T; t0 += chunk) {
            const int n = (T - t0) < chunk ? (T - t0) : chunk;
            s = stack_enqueue(L, n_layers, W, bias, blobs, x + (size_t)t0 * L->shape.d, n, eps, st);
            L->tiled_tokens = -1;  // the layers' routing went to the workspace in turn
            if (s != STRATA_OK) return s;
        }
        return STRATA_OK;
    }
    // decode sizes: replay a captured graph while the arguments are unchanged
    std::vector<const void *> key;
    key.reserve(3 * n_layers + 4);
    for (int l = 0; l < n_layers; ++l) {
        key.push_back(W[l]);
        key.push_back(bias ? bias[l] : nullptr);
        key.push_back(blobs[l]);
    }
    key.push_back(x);
    key.push_back(reinterpret_cast<const void *>((uintptr_t)T));
    uint32_t epsbits;
    memcpy(&epsbits, &eps, 4);
    key.push_back(reinterpret_cast<const void *>((uintptr_t)epsbits));
    if (!L->graph.exec || L->graph.key != key) {
        if (L->graph.exec) {
            cudaGraphExecDestroy(L->graph.exec);
            L->graph.exec = nullptr;
        }
        // capture on the library's own stream (the caller's may be the legacy
        // default stream, which cannot be captured); the graph is launched on
        // the caller's stream
        if (!L->capture_stream) CUDA_TRY(cudaStreamCreateWithFlags(&L->capture_stream, cudaStreamNonBlocking));
        CUDA_TRY(cudaStreamBeginCapture(L->capture_stream, cudaStreamCaptureModeThreadLocal));
        s = stack_enqueue(L, n_layers, W, bias, blobs, x, T, eps, L->capture_stream);
        cudaGraph_t g = nullptr;
        cudaError_t ce = cudaStreamEndCapture(L->capture_stream, &g);
        if (s != STRATA_OK) {
            if (g) cudaGraphDestroy(g);
            return s;
        }
        if (ce != cudaSuccess) return fail(STRATA_ERR_CUDA, "stream capture failed: %s", cudaGetErrorString(ce));
        ce = cudaGraphInstantiate(&L->graph.exec, g, 0);
        cudaGraphDestroy(g);
        if (ce != cudaSuccess) {
            L->graph.exec = nullptr;
            return fail(STRATA_ERR_CUDA, "graph instantiate failed: %s", cudaGetErrorString(ce));
        }
        L->graph.key = key;
    }
    CUDA_TRY(cudaGraphLaunch(L->graph.exec, st));
    return STRATA_OK;
}

extern "C" strata_status strata_moe_check_status(strata_moe_layer L) {
    if (!L) return fail(STRATA_ERR_INVALID_ARG, "layer is NULL");
    CUDA_TRY(cudaDeviceSynchronize());
    uint32_t w = 0;
    CUDA_TRY(cudaMemcpy(&w, L->ws.status, 4, cudaMemcpyDeviceToHost));
    CUDA_TRY(cudaMemset(L->ws.status, 0, 4));
    if (w & kStatusTimeout) {
        cudaMemset(L->ws.sync, 0, (size_t)(2 + L->shape.E) * 4);  // counters of an unwound launch
        return fail(STRATA_ERR_TIMEOUT, "a device wait exceeded its time limit");
    }
    if (w & kStatusBounds) return fail(STRATA_ERR_BOUNDS, "a bounds check of the checked build failed");
    return STRATA_OK;
}

extern "C" strata_status strata_selftest_wait_timeout(uint64_t timeout_ns, strata_stream_t stream) {
    if (timeout_ns < 1000ull || timeout_ns > 10000000000ull)
        return fail(STRATA_ERR_INVALID_ARG, "timeout_ns must be in 1e3..1e10");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint32_t *status = nullptr;
    CUDA_TRY(cudaMalloc(&status, 4));
    cudaMemsetAsync(status, 0, 4, st);
    launch_wait_selftest(status, timeout_ns, st);
    strata_status s = check_launch("self-test kernel");
    uint32_t w = 0;
    if (s == STRATA_OK && cudaMemcpyAsync(&w, status, 4, cudaMemcpyDeviceToHost, st) == cudaSuccess &&
        cudaStreamSynchronize(st) == cudaSuccess) {
        s = (w & kStatusTimeout) ? fail(STRATA_ERR_TIMEOUT, "self-test wait timed out as intended") : STRATA_OK;
    } else if (s == STRATA_OK) {
        s = fail(STRATA_ERR_CUDA, "self-test readback failed");
    }
    cudaFree(status);
    return s;
}

extern "C" int32_t strata_is_checked_build(void) { return kChecked ? 1 : 0; }

extern "C" strata_status strata_selftest_bounds_check(strata_stream_t stream) {
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint32_t *status = nullptr;
    CUDA_TRY(cudaMalloc(&status, 4));
    cudaMemsetAsync(status, 0, 4, st);
    launch_bounds_selftest(status, st);
    strata_status s = check_launch("bounds self-test kernel");
    uint32_t w = 0;
    if (s == STRATA_OK && cudaMemcpyAsync(&w, status, 4, cudaMemcpyDeviceToHost, st) == cudaSuccess &&
        cudaStreamSynchronize(st) == cudaSuccess) {
        s = (w & kStatusBounds) ? fail(STRATA_ERR_BOUNDS, "self-test index out of range, recorded as intended")
                                : STRATA_OK;
    } else if (s == STRATA_OK) {
        s = fail(STRATA_ERR_CUDA, "self-test readback failed");
    }
    cudaFree(status);
    return s;
}

// ------------------------------------------------------------ packers
// Tile (p, s) of a [rows x K] matrix -- rows 64p.., columns 64s.. -- goes to
// dst + p * panel_stride + s * slice_stride. Column c = 16j + 8s + 2t + h of
// a tile row: 2-bit codes in word t at bit 16h + 8s + 6 - 2j (four words);
// 4-bit codes in word 2t + j/2 at bit 16h + 8(j%2) + 4s (eight words).
static void pack_matrix_host(const uint8_t *codes, const uint16_t *scales, int rows, int K, int bits, uint8_t *dst,
                             size_t panel_stride, size_t slice_stride) {
    const int nw = bits == 4 ? 8 : 4;
    const size_t soff = bits == 4 ? Qn<4>::kScaleOffset : Qn<2>::kScaleOffset;
    for (int p = 0; p < rows / STRATA_Q2_TILE_ROWS; ++p)
        for (int s = 0; s < K / STRATA_Q2_TILE_COLS; ++s) {
            uint8_t *t = dst + (size_t)p * panel_stride + (size_t)s * slice_stride;
            for (int i = 0; i < STRATA_Q2_TILE_ROWS; ++i) {
                const int r = p * STRATA_Q2_TILE_ROWS + i;
                uint32_t w[8] = {0, 0, 0, 0, 0, 0, 0, 0};
                for (int c = 0; c < 64; ++c) {
                    const uint32_t v = codes[(size_t)r * K + 64 * s + c];
                    const int j = c / 16, sh = (c / 8) % 2, tq = (c % 8) / 2, h = c % 2;
                    if (bits == 4)
                        w[2 * tq + j / 2] |= (v & 15u) << (16 * h + 8 * (j % 2) + 4 * sh);
                    else
                        w[tq] |= (v & 3u) << (16 * h + 8 * sh + 6 - 2 * j);
                }
                for (int q = 0; q < nw; ++q)
                    for (int b = 0; b < 4; ++b) t[4 * nw * i + 4 * q + b] = (uint8_t)(w[q] >> (8 * b));
                for (int b = 0; b < 2; ++b) {
                    const uint16_t sv = scales[(size_t)r * (K / 32) + 2 * s + b];
                    t[soff + 4 * i + 2 * b] = (uint8_t)(sv & 0xff);
                    t[soff + 4 * i + 2 * b + 1] = (uint8_t)(sv >> 8);
                }
            }
        }
}

static strata_status check_codes(const uint8_t *codes, size_t n, int bits) {
    const unsigned top = (1u << bits) - 1u;
    for (size_t i = 0; i < n; ++i)
        if (codes[i] > top)
            return fail(STRATA_ERR_BAD_BLOB, "code %u at index %zu is not in 0..%u", codes[i], i, top);
    return STRATA_OK;
}

static strata_status pack_lone_matrix(const uint8_t *codes, const uint16_t *scales, int32_t rows, int32_t K,
                                      int bits, void *dst) {
    if (!codes || !scales || !dst) return fail(STRATA_ERR_INVALID_ARG, "NULL pointer");
    if (rows <= 0 || K <= 0 || rows % STRATA_Q2_TILE_ROWS || K % STRATA_Q2_TILE_COLS)
        return fail(STRATA_ERR_INVALID_ARG, "rows and K must be multiples of 64 (got %d x %d)", rows, K);
    strata_status s = check_codes(codes, (size_t)rows * K, bits);
    if (s != STRATA_OK) return s;
    const size_t tb = bits == 4 ? STRATA_Q4_TILE_BYTES : STRATA_Q2_TILE_BYTES;
    pack_matrix_host(codes, scales, rows, K, bits, static_cast<uint8_t *>(dst), (size_t)(K / STRATA_Q2_TILE_COLS) * tb,
                     tb);
    return STRATA_OK;
}

extern "C" strata_status strata_q2_pack(const uint8_t *codes, const uint16_t *scales, int32_t rows, int32_t K,
                                        void *dst) {
    return pack_lone_matrix(codes, scales, rows, K, 2, dst);
}

extern "C" strata_status strata_q4_pack(const uint8_t *codes, const uint16_t *scales, int32_t rows, int32_t K,
                                        void *dst) {
    return pack_lone_matrix(codes, scales, rows, K, 4, dst);
}

extern "C" strata_status strata_moe_pack_expert(const strata_moe_desc *desc, const uint8_t *gc, const uint16_t *gs,
                                                const uint8_t *uc, const uint16_t *us, const uint8_t *dc,
                                                const uint16_t *ds, void *dst) {
    strata_status s = validate_desc(desc);
    if (s != STRATA_OK) return s;
    if (!gc || !gs || !uc || !us || !dc || !ds || !dst) return fail(STRATA_ERR_INVALID_ARG, "NULL pointer");
    const Shape sh = shape_of(desc);
    const size_t n = (size_t)sh.d * sh.f;
    if ((s = check_codes(gc, n, sh.bits)) != STRATA_OK || (s = check_codes(uc, n, sh.bits)) != STRATA_OK ||
        (s = check_codes(dc, n, sh.bits)) != STRATA_OK)
        return s;
    uint8_t *b = static_cast<uint8_t *>(dst);
    const ExpertStrides x = expert_strides(sh);
    pack_matrix_host(gc, gs, sh.f, sh.d, sh.bits, b, x.gu_panel, x.gu_slice);
    pack_matrix_host(uc, us, sh.f, sh.d, sh.bits, b + tile_bytes(sh), x.gu_panel, x.gu_slice);
    pack_matrix_host(dc, ds, sh.d, sh.f, sh.bits, b + down_section_offset(sh), x.dn_panel, x.dn_slice);
    return STRATA_OK;
}

extern "C" strata_status strata_moe_pack_expert_device(const strata_moe_desc *desc, const uint8_t *gc,
                                                       const uint16_t *gs, const uint8_t *uc, const uint16_t *us,
                                                       const uint8_t *dc, const uint16_t *ds, void *dst,
                                                       strata_stream_t stream) {
    strata_status s = validate_desc(desc);
    if (s != STRATA_OK) return s;
    if (!gc || !gs || !uc || !us || !dc || !ds || !dst) return fail(STRATA_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned16(dst)) return fail(STRATA_ERR_BAD_BLOB, "dst must be 16-byte aligned");
    const Shape sh = shape_of(desc);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *b = static_cast<uint8_t *>(dst);
    const ExpertStrides x = expert_strides(sh);
    launch_pack_matrix_device(gc, gs, sh.f, sh.d, sh.bits, b, x.gu_panel, x.gu_slice, st);
    launch_pack_matrix_device(uc, us, sh.f, sh.d, sh.bits, b + tile_bytes(sh), x.gu_panel, x.gu_slice, st);
    launch_pack_matrix_device(dc, ds, sh.d, sh.f, sh.bits, b + down_section_offset(sh), x.dn_panel, x.dn_slice, st);
    return check_launch("pack kernels");
}
