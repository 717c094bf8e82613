// route_noalloc.cu -- the routing call without any allocation.
//
// strata_moe_route needs a layer handle, and creating one allocates the
// layer's workspace. Some callers cannot allocate at the moment they route:
// one whose device memory has all been handed to another allocator (a
// caching pool that owns every free byte), or a serving loop that must not
// call cudaMalloc / cudaFree because those calls can synchronise the whole
// device and stall the work of every other stream. This entry point runs the
// same routing kernels as strata_moe_route (router GEMV, softmax top-k,
// per-expert lists) with their scratch in a fixed-size array in device
// memory that belongs to this translation unit, and writes the routing
// straight into the caller's buffers.
//
// Scratch: one static device array of kNoallocScratchBytes per device, enough
// for n_tokens <= STRATA_NOALLOC_MAX_TOKENS, n_experts <= 1024 and
// top_k <= 32 (the limits the descriptor already enforces for E and k).
// Nothing in it has to start at zero: every kernel of the routing writes
// each scratch word it later reads, in this call.
//
// Set-up: the first call on a device (with that device current) looks up the
// array's device address with cudaGetSymbolAddress, under a lock; the address
// is kept per device ordinal together with the context it belongs to, and is
// looked up again when the current context differs (after a device reset).
// That first call can load the module, so it should be made before any
// stream capture that will contain the call.
//
// Concurrency: all calls on one device share the one array. Two calls whose
// work can overlap on the device (different streams without an ordering
// between them) race on it and give undefined routing; callers serialise
// them, e.g. by issuing them on one stream.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "abi_internal.h"
#include "kernels.h"

namespace {

using strata::kGemm1N;
using strata::kGemm2N;

constexpr int kMaxT = STRATA_NOALLOC_MAX_TOKENS;
constexpr int kMaxE = 1024;
constexpr int kMaxK = 32;
constexpr int kMaxPairs = kMaxT * kMaxK;
constexpr int kMaxTiles1 = (kMaxPairs + kGemm1N - 1) / kGemm1N + kMaxE;
constexpr int kMaxTiles2 = (kMaxPairs + kGemm2N - 1) / kGemm2N + kMaxE;

constexpr size_t up256(size_t v) { return (v + 255) & ~(size_t)255; }

// byte offsets of the scratch buffers (the largest sizes this call accepts)
constexpr size_t kOffMeta = 0;
constexpr size_t kOffLogits = kOffMeta + up256(64 * 4);
constexpr size_t kOffBlkCounts = kOffLogits + up256((size_t)kMaxT * kMaxE * 4);
constexpr size_t kOffCounts = kOffBlkCounts + up256((size_t)kMaxE * 4);  // one 256-token block
constexpr size_t kOffPairW = kOffCounts + up256((size_t)kMaxE * 4);
constexpr size_t kOffPairOf = kOffPairW + up256((size_t)kMaxPairs * 4);
constexpr size_t kOffTiles1 = kOffPairOf + up256((size_t)kMaxPairs * 4);
constexpr size_t kOffTiles2 = kOffTiles1 + up256((size_t)kMaxTiles1 * 16);
constexpr size_t kNoallocScratchUsed = kOffTiles2 + up256((size_t)kMaxTiles2 * 16);
constexpr size_t kNoallocScratchBytes = STRATA_NOALLOC_SCRATCH_BYTES;
static_assert(kNoallocScratchUsed <= kNoallocScratchBytes, "routing scratch does not fit");
static_assert(kMaxT <= strata::kRouteBlock, "one list block must cover the tokens");

__device__ __align__(256) static unsigned char g_route_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
struct ScratchEntry {
    CUcontext ctx;  // context the address belongs to
    void *addr;
};
ScratchEntry g_scratch[kMaxDevices];

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

CtxGetCurrentFn ctx_get_current() {
    static CtxGetCurrentFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    }
    return fn;
}

// Device address of this device's scratch in the current context. It is
// looked up once per (device, context): after a cudaDeviceReset the device's
// primary context is a new one, the old address is stale, and it is looked
// up again.
strata_status scratch_of_current_device(unsigned char **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return strata_set_error(STRATA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices)
        return strata_set_error(STRATA_ERR_UNSUPPORTED, "device ordinal %d beyond %d", dev, kMaxDevices - 1);
    CtxGetCurrentFn get = ctx_get_current();
    if (!get) return strata_set_error(STRATA_ERR_CUDA, "cuCtxGetCurrent is not available");
    CUcontext ctx = nullptr;  // null while no context is current on this thread yet
    if (get(&ctx) != CUDA_SUCCESS) return strata_set_error(STRATA_ERR_CUDA, "cannot read the current CUDA context");
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    ScratchEntry &ent = g_scratch[dev];
    if (!ent.addr || !ctx || ent.ctx != ctx) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_route_scratch);  // makes the primary context current if none is
        if (e != cudaSuccess || !p)
            return strata_set_error(STRATA_ERR_CUDA, "cudaGetSymbolAddress of the routing scratch: %s",
                                    cudaGetErrorString(e));
        if (get(&ctx) != CUDA_SUCCESS || !ctx)
            return strata_set_error(STRATA_ERR_CUDA, "cannot read the current CUDA context");
        ent.ctx = ctx;
        ent.addr = p;
    }
    *out = static_cast<unsigned char *>(ent.addr);
    return STRATA_OK;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" strata_status strata_moe_route_noalloc(const strata_moe_desc *desc, const void *x_bf16,
                                                  const float *router_w, int32_t n_tokens, int32_t *topk_idx,
                                                  float *topk_w, int32_t *expert_offsets, int32_t *token_list,
                                                  int32_t *pair_slot, strata_stream_t stream) {
    if (!desc) return strata_set_error(STRATA_ERR_INVALID_ARG, "desc is NULL");
    // max_tokens and flags play no part in this call: check the rest only
    strata_moe_desc checked = *desc;
    checked.max_tokens = 1;
    checked.flags = 0;
    strata_status s = strata_check_desc(&checked);
    if (s != STRATA_OK) return s;
    if (n_tokens < 0) return strata_set_error(STRATA_ERR_INVALID_ARG, "n_tokens < 0");
    if (n_tokens > kMaxT)
        return strata_set_error(STRATA_ERR_TOO_MANY_TOKENS,
                                "n_tokens %d > %d: the allocation-free routing scratch holds at most %d tokens",
                                n_tokens, kMaxT, kMaxT);
    if (!x_bf16 || !router_w || !topk_idx || !topk_w || !expert_offsets || !token_list || !pair_slot)
        return strata_set_error(STRATA_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned(x_bf16, 16) || !aligned(router_w, 16))
        return strata_set_error(STRATA_ERR_INVALID_ARG, "x and router_w must be 16-byte aligned");
    if (!aligned(topk_idx, 4) || !aligned(topk_w, 4) || !aligned(expert_offsets, 4) || !aligned(token_list, 4) ||
        !aligned(pair_slot, 4))
        return strata_set_error(STRATA_ERR_INVALID_ARG, "routing outputs must be 4-byte aligned");
    unsigned char *base = nullptr;
    if ((s = scratch_of_current_device(&base)) != STRATA_OK) return s;
    if (n_tokens == 0) return STRATA_OK;

    const strata::Shape sh{desc->d_model, desc->d_ff, desc->n_experts, desc->top_k,
                           desc->weight_format == STRATA_FMT_Q4_0_TILED ? 4 : 2};
    const int P = n_tokens * sh.k;
    strata::Workspace ws{};
    ws.meta = reinterpret_cast<int32_t *>(base + kOffMeta);
    ws.logits = reinterpret_cast<float *>(base + kOffLogits);
    ws.blk_counts = reinterpret_cast<int32_t *>(base + kOffBlkCounts);
    ws.counts = reinterpret_cast<int32_t *>(base + kOffCounts);
    ws.pair_w = reinterpret_cast<float *>(base + kOffPairW);
    ws.pair_of = reinterpret_cast<int32_t *>(base + kOffPairOf);
    ws.tiles1 = reinterpret_cast<int4 *>(base + kOffTiles1);
    ws.tiles2 = reinterpret_cast<int4 *>(base + kOffTiles2);
    ws.topk_idx = topk_idx;
    ws.topk_w = topk_w;
    ws.offsets = expert_offsets;
    ws.token_list = token_list;
    ws.pair_slot = pair_slot;
    const int max_tiles1 = (P + kGemm1N - 1) / kGemm1N + sh.E;
    const int max_tiles2 = (P + kGemm2N - 1) / kGemm2N + sh.E;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    strata::launch_router_gemv(x_bf16, router_w, desc->router_bias, ws.logits, n_tokens, sh, st);
    strata::launch_route_large(ws, n_tokens, max_tiles1, max_tiles2, sh, st);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return strata_set_error(STRATA_ERR_CUDA, "routing kernels: %s", cudaGetErrorString(e));
    return STRATA_OK;
}
