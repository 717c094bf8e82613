// topk.cuh -- one warp's softmax top-k of one token's logits (shared by the
// one-launch decode kernel and the prefill routing kernels).
//
// Selection key: the fp32 logit, descending, ties to the lower expert index
// (the layer's routing rule; 10 experts per token, "Strata：把 125B 大模型塞进
// 12GB 显卡…", 核心思路).
#pragma once

#include "common.cuh"

namespace strata {

// monotone map of a float to uint32 (+0 and -0 both map to 0x80000000);
// every finite or infinite value maps above 0, the "taken" marker
STRATA_DEV uint32_t ordered_key(float v) {
    uint32_t u = __float_as_uint(v + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
STRATA_DEV float key_value(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// ------------------------------------------------------------ top-k
// One warp, the experts e0 .. e1-1 of one token's logit row (e0 % 4 == 0,
// E % 4 == 0 so every float4 read stays inside the row). Lane l holds the
// logits of experts e0 + KPL*l .. e0 + KPL*l + KPL - 1 as ordered keys,
// sorted in registers (bitonic network, key descending, then expert
// ascending). Among equal keys the lowest lane holds the lowest expert index,
// so each of the k rounds takes the warp max of the lanes' heads and the
// lowest lane holding it (ballot), which pops its head. emit(j, key, expert)
// runs on lane 0 for the j-th best, j < k; past the last expert of the range
// it emits key 0 (below every real key) and expert -1.
template <int KPL, typename Emit>
STRATA_DEV void range_topk(const float *row, int e0, int e1, int k, Emit emit) {
    const int lane = threadIdx.x & 31;
    uint32_t key[KPL];
    int pos[KPL];
    if constexpr (KPL >= 4) {
#pragma unroll
        for (int i = 0; i < KPL; i += 4) {
            const int e = e0 + KPL * lane + i;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (e < e1) v = __ldcg(reinterpret_cast<const float4 *>(row + e));
            const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                key[i + q] = e + q < e1 ? ordered_key(vv[q]) : 0u;  // 0: below every real key
                pos[i + q] = i + q;
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < KPL; ++i) {
            const int e = e0 + KPL * lane + i;
            key[i] = e < e1 ? ordered_key(__ldcg(row + e)) : 0u;
            pos[i] = i;
        }
    }
#pragma unroll
    for (int size = 2; size <= KPL; size <<= 1)
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1)
#pragma unroll
            for (int i = 0; i < KPL; ++i) {
                const int j = i ^ stride;
                if (j > i) {
                    // ascending blocks reversed: the network sorts descending by (key, -position)
                    const bool desc = (i & size) == 0;
                    const bool jfirst = key[j] > key[i] || (key[j] == key[i] && pos[j] < pos[i]);
                    const bool sw = desc ? jfirst : !jfirst;
                    const uint32_t tk = key[i];
                    const int tp = pos[i];
                    key[i] = sw ? key[j] : tk;
                    pos[i] = sw ? pos[j] : tp;
                    key[j] = sw ? tk : key[j];
                    pos[j] = sw ? tp : pos[j];
                }
            }
    for (int j = 0; j < k; ++j) {
        const uint32_t m = __reduce_max_sync(0xffffffffu, key[0]);
        const int wl = __ffs(__ballot_sync(0xffffffffu, key[0] == m)) - 1;
        const int wp = __shfl_sync(0xffffffffu, pos[0], wl);
        if (lane == 0) emit(j, m, m ? e0 + KPL * wl + wp : -1);
        if (lane == wl) {
#pragma unroll
            for (int i = 0; i + 1 < KPL; ++i) {
                key[i] = key[i + 1];
                pos[i] = pos[i + 1];
            }
            key[KPL - 1] = 0u;
        }
    }
}

// One warp, one token, all E experts: the k best as expert indices and logits.
template <int KPL>
STRATA_DEV void token_topk(const float *logits, int t, int E, int k, int *sel_idx, float *sel_val) {
    range_topk<KPL>(logits + (size_t)t * E, 0, E, k, [&](int j, uint32_t key, int e) {
        sel_idx[j] = e;
        sel_val[j] = key_value(key);
    });
}

// One warp merges G candidate lists (list g: keys ckey[g * k + j], experts
// cidx[g * k + j], j < k, each in selection order, the lists covering
// ascending expert ranges) into the k best of the token. Equal keys go to the
// lowest list, which holds the lowest experts, so the result equals a
// single-warp selection over the whole row.
STRATA_DEV void merge_topk(const uint32_t *ckey, const int *cidx, int G, int k, int *sel_idx, float *sel_val) {
    const int lane = threadIdx.x & 31;
    int head = 0;
    uint32_t hk = lane < G ? ckey[lane * k] : 0u;
    for (int j = 0; j < k; ++j) {
        const uint32_t m = __reduce_max_sync(0xffffffffu, hk);
        const int wl = __ffs(__ballot_sync(0xffffffffu, lane < G && hk == m)) - 1;
        const int e = __shfl_sync(0xffffffffu, lane < G && head < k ? cidx[lane * k + head] : -1, wl);
        if (lane == 0) {
            sel_idx[j] = e;
            sel_val[j] = key_value(m);
        }
        if (lane == wl) {
            ++head;
            hk = head < k ? ckey[lane * k + head] : 0u;
        }
    }
}

}  // namespace strata
