// common.cuh -- shared device helpers of the sm_100a kernels: status word,
// time-bounded waits, mbarriers, bulk / tensor (TMA) copies and tcgen05
// (tensor memory + 5th-generation MMA) wrappers as inline PTX.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define STRATA_DEV __device__ __forceinline__

namespace strata {

// ---------------------------------------------------------------- status
// Device status word: 0 = OK; bit 0 = a bounded wait ran out; bit 1 = a
// bounds check of the checked build (STRATA_CHECKED) failed.
// Every spin-wait below gives up after kWaitLimitNs and sets the word.
enum : uint32_t { kStatusTimeout = 1u, kStatusBounds = 2u };
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

STRATA_DEV uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

STRATA_DEV void set_status(uint32_t *status, uint32_t bits) {
    if (status) atomicOr(status, bits);
}

// Bounds checks of the checked build: compiled with -DSTRATA_CHECKED, every
// index the kernels take from data (an expert, a token, a pair, a list
// position, a tile) is tested before use; a bad one is recorded in the status
// word and replaced by `fallback` (or its access skipped), so the kernel
// neither faults nor traps. In the normal build the checks compile away.
#ifdef STRATA_CHECKED
constexpr bool kChecked = true;
#else
constexpr bool kChecked = false;
#endif

STRATA_DEV bool in_bounds(long long v, long long hi, uint32_t *status) {
    if (kChecked && (v < 0 || v >= hi)) {
        set_status(status, kStatusBounds);
        return false;
    }
    return true;
}

STRATA_DEV int checked_index(int v, int hi, int fallback, uint32_t *status) {
    return in_bounds(v, hi, status) ? v : fallback;
}

STRATA_DEV uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
STRATA_DEV void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

STRATA_DEV void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

STRATA_DEV void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

STRATA_DEV void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

STRATA_DEV bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait until the barrier completes the phase of the given parity. Gives up
// after kWaitLimitNs (or at once when *abort is set), sets the status word
// and *abort, and returns false.
STRATA_DEV bool mbar_wait(uint64_t *bar, uint32_t parity, uint32_t *status, volatile int *abort,
                          uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    uint64_t t0 = globaltimer();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63u) == 0) {
            if (abort && *abort) return false;
            if (globaltimer() - t0 > limit_ns) {
                set_status(status, kStatusTimeout);
                if (abort) *abort = 1;
                return false;
            }
        }
    }
}

// ---------------------------------------------------------------- copies
// 1-D bulk copy global -> shared, completion counted on `bar` (bytes).
STRATA_DEV void bulk_g2s(void *dst_smem, const void *src_gmem, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// 4-byte asynchronous global -> shared copy (the issuing thread does not
// wait); cp_async_wait_all() by the same thread waits for its copies.
STRATA_DEV void cp_async4(void *dst_smem, const void *src_gmem) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst_smem)), "l"(src_gmem) : "memory");
}
STRATA_DEV void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Ask L2 to fetch [src, src + bytes) from memory (no completion signal).
STRATA_DEV void prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// 2-D tiled tensor copy global -> shared (no multicast).
STRATA_DEV void tma_load_2d(void *dst_smem, const CUtensorMap *map, int32_t x, int32_t y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(smem_u32(dst_smem)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

STRATA_DEV void prefetch_tmap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Programmatic dependent launch: wait until the grids this launch depends on
// have completed and their memory is visible (a no-op for a launch without
// the programmatic-serialization attribute), and let the launches that depend
// on this grid start once every CTA has signalled or exited.
STRATA_DEV void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
STRATA_DEV void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// generic-proxy smem writes -> visible to the async proxy (tensor core, TMA)
STRATA_DEV void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ---------------------------------------------------------------- tcgen05
STRATA_DEV void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
STRATA_DEV void tmem_relinquish() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory"); }
STRATA_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
STRATA_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
STRATA_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (fp16/bf16 in, fp32 accumulate)
STRATA_DEV void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// arrive on `bar` once all previously issued tcgen05.mma of this thread finish
STRATA_DEV void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// 32 lanes x 32 bits, 16 consecutive columns per thread
STRATA_DEV void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
STRATA_DEV void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, 8-row
// groups 1024 bytes apart (rows of 64 fp16 = 128 bytes).
STRATA_DEV uint64_t umma_desc_sw128(const void *smem_tile) {
    uint64_t a = smem_u32(smem_tile);
    return ((a >> 4) & 0x3FFFull) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: A, B fp16, D fp32, both K-major.
__host__ __device__ constexpr uint32_t umma_idesc_f16(int M, int N) {
    return (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------- misc
STRATA_DEV float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// silu(g) = g / (1 + e^-g) with the hardware exponential and a fast divide (a
// few fp32 ulp; both SwiGLU epilogues round the product to fp16 next)
STRATA_DEV float silu_fast(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// Power-of-two scale of one token's activations for the fp16 operands: 1 when
// the token's largest |x| is in [2^-4, 2^4] (the arithmetic is then the
// unscaled one), else s = 2^e with amax * s in [1, 2) (e clamped to [-30, 30],
// so that 1 / s^2 stays a normal fp32 multiplier; amax == 0 gives 1).
// Multiplying by s, and later by 1 / s or 1 / s^2, is exact in fp32, so the
// scaled fp16 operands keep bf16's dynamic range: every element within 2^-14
// of the token's largest is a normal fp16 number.
STRATA_DEV float pow2_scale(float amax) {
    if (amax >= 0.0625f && amax <= 16.f) return 1.f;  // already in range: no scaling
    const uint32_t ex = (__float_as_uint(amax) >> 23) & 0xffu;  // amax >= 0
    int e = amax > 0.f ? 127 - (int)ex : 0;
    e = e < -30 ? -30 : (e > 30 ? 30 : e);
    return __uint_as_float((uint32_t)(127 + e) << 23);
}
// 1 / s for s = pow2_scale(...) (a power of two): the exponent reflected, exact.
STRATA_DEV float pow2_inverse(float s) { return __uint_as_float((254u << 23) - __float_as_uint(s)); }

}  // namespace strata
