// kernels.h -- host-side launchers of the sm_100a kernels (internal).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace strata {

// Workspace of one layer handle (all device pointers, carved from one
// allocation). Sizes are for max_tokens tokens (T) and top_k (k).
struct Workspace {
    uint32_t *status;     // [1]  device status word
    int32_t *meta;        // [16] n_active, n_tiles1, n_tiles2, n_tokens, ...
    float *logits;        // [T * E]
    int32_t *topk_idx;    // [T * k]
    float *topk_w;        // [T * k]
    int32_t *counts;      // [E]
    int32_t *offsets;     // [E + 1]
    int32_t *token_list;  // [T * k]
    int32_t *pair_slot;   // [T * k]
    float *pair_w;        // [T * k]
    int32_t *pair_of;     // [T * k]   (t, j) -> index in the sorted pair list
    int32_t *blk_counts;  // [nblk * E] per 256-token block (prefill lists)
    int32_t *act;         // [E] active experts (decode path)
    float *lpart;         // [16 * E * 4]        fused decode: router logits [T][E]
    void *xp;             // fp16 [T*k * d]       gathered expert inputs (prefill), token scale applied
    float *pair_s;        // [T * k]  power-of-two scale of each sorted pair's token (prefill)
    float *tok_s;         // [T]      power-of-two scale of each token (prefill)
    void *hbuf;           // fp16 [T*k * f]       SwiGLU outputs (prefill)
    int4 *tiles1;         // gate/up GEMM tiles {expert, pair_start, n, 0}
    int4 *tiles2;         // down GEMM tiles
    void *xn;             // bf16 [T * d]         stack: normalised input
    void *w_hi, *w_lo;    // bf16 [E * d] each    prefill router: bf16 split of W_r
    uint32_t *sync;       // [2]     fused decode: grid barrier, exit count
};

// meta[] slots
enum { META_N_ACTIVE = 0, META_N_TILES1 = 1, META_N_TILES2 = 2, META_N_TOKENS = 3 };

constexpr int kRouteBlock = 256;      // tokens per block of the prefill lists
constexpr int kDecMaxT = 16;          // largest token count of the streaming path
constexpr int kGemm1N = 128;          // gate/up GEMM: max tokens per tile
constexpr int kGemm2N = 256;          // down GEMM: max tokens per tile

struct Shape {
    int d, f, E, k;
    int bits;  // code width of the expert weights: 2 or 4
};

struct TmaMaps {
    CUtensorMap m[5];  // box rows 16, 32, 64, 128, 256
};

// prefill router on the tensor cores: W_hi / W_lo [E x d] (boxes 64 x 128),
// x [T x d] (box 64 x 256), bf16, 128-byte swizzle
struct RouterMaps {
    CUtensorMap w_hi, w_lo, x;
};

// --- routing
void launch_router_gemv(const void *x, const float *W, const float *bias, float *logits, int T, const Shape &s,
                        cudaStream_t st);
// prefill sizes: splits W into bf16 hi/lo (ws.w_hi, ws.w_lo), then the tensor-core GEMM
void launch_router_tc(const Workspace &ws, const RouterMaps &maps, const float *W, const float *bias, float *logits,
                      int T, const Shape &s, int num_sms, cudaStream_t st);
cudaError_t init_router_attributes(int max_smem);
// x_scale_src: the bf16 tokens whose power-of-two scales go to ws.tok_s, or
// nullptr (routing only)
void launch_route_large(const Workspace &ws, int T, int max_tiles1, int max_tiles2, const Shape &s,
                        cudaStream_t st, const void *x_scale_src = nullptr);
void launch_gather_xp(const Workspace &ws, const void *x, int T, const Shape &s, cudaStream_t st);

// --- fused decode layer (T <= 16, one cooperative launch)
bool decode_fused_supported(const Shape &s, int T, int max_smem, int num_sms);
// raise the kernels' shared-memory limits to what this shape needs (layer creation)
cudaError_t init_fused_attributes(const Shape &s, int max_tokens, int max_smem, int num_sms);
cudaError_t launch_decode_fused(const Workspace &ws, const void *x, const float *W, const float *bias,
                                const uint8_t *blob, float *y, bool accumulate, bool rms, float eps, int T,
                                const Shape &s, int num_sms, int max_smem, cudaStream_t st, cudaEvent_t *ev);

// --- prefill experts (tensor cores)
void launch_expert_gemm1(const Workspace &ws, const uint8_t *blob, const TmaMaps &maps, int max_tiles, int T,
                         const Shape &s, int num_sms, cudaStream_t st);
// writes w * W_down h per pair into ws.xp (fp16 [pairs x d]); launch_combine sums them into y
void launch_expert_gemm2(const Workspace &ws, const uint8_t *blob, float *y, const TmaMaps &maps, int max_tiles, int T,
                         const Shape &s, int num_sms, cudaStream_t st);
void launch_combine(const Workspace &ws, float *y, bool accumulate, int T, const Shape &s, cudaStream_t st);

// --- misc
void launch_rmsnorm_bf16(const float *x, void *out, int T, int d, float eps, cudaStream_t st);
void launch_pack_matrix_device(const uint8_t *codes, const uint16_t *scales, int rows, int K, int bits, uint8_t *dst,
                               size_t panel_stride, size_t slice_stride, cudaStream_t st);
void launch_wait_selftest(uint32_t *status, uint64_t timeout_ns, cudaStream_t st);
// one index one past the end of a 16-entry array, tested with in_bounds (the
// access is skipped): the status word records it in the checked build only
void launch_bounds_selftest(uint32_t *status, cudaStream_t st);

size_t expert_bytes(const Shape &s);

// Tiles: 64 rows x 64 columns, codes then scales. 2-bit: 16 code bytes per
// row; 4-bit: 32. Qn<BITS> gives a format's sizes at compile time.
constexpr int kTileRows = 64;
template <int BITS>
struct Qn {
    static constexpr int kRowBytes = 64 * BITS / 8;                // code bytes of one tile row
    static constexpr int kScaleOffset = 64 * kRowBytes;            // 1024 or 2048
    static constexpr int kTileBytes = kScaleOffset + 64 * 4;       // 1280 or 2304
};
constexpr int kTileBytes = Qn<2>::kTileBytes;
constexpr int kTileScaleOffset = Qn<2>::kScaleOffset;
inline size_t tile_bytes(const Shape &s) { return s.bits == 4 ? Qn<4>::kTileBytes : Qn<2>::kTileBytes; }

// Byte strides between the tiles of an expert's matrices: gate/up tiles
// (f-panel p, d-slice s) at p * gu_panel + s * gu_slice (gate, then up one
// tile later); down tiles (d-panel p, f-slice s) at p * dn_panel + s * dn_slice.
struct ExpertStrides {
    size_t gu_panel, gu_slice, dn_panel, dn_slice;
};
inline ExpertStrides expert_strides(const Shape &s) {
    const size_t tb = tile_bytes(s);
    return ExpertStrides{(size_t)(s.d / 64) * 2 * tb, 2 * tb, tb, (size_t)(s.d / 64) * tb};
}

size_t down_section_offset(const Shape &s);

}  // namespace strata
