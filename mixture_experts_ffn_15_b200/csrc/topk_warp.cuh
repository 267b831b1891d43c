// Top-k selection and routing weights of ONE token by ONE warp, shared by the
// single-CTA router and the routed decode FFN so that both give the same bits.
//
// "Gemma 4 MoE: re-enable fused com.microsoft::MoE op - #326", "Attribute set":
// k = top_k, normalize_routing_weights.  The chosen experts are the k largest
// (logit + bias) in descending order, equal values to the lower expert index; the
// weights are the softmax over all E experts, renormalised over the chosen k
// (normalize = 1, which equals the softmax over the chosen k) or kept as they are.
#pragma once

#include <math.h>

#include "common.cuh"

namespace moe {

constexpr int kWarpTopkVals = kMaxExperts / 32;   // logits held per lane

// float -> unsigned with the same order (larger float, larger key)
__device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

struct WarpTopk {
    int idx;     // lane j < k: the j-th chosen expert
    float w;     // lane j < k: its routing weight
    int flags;   // every lane: bit 1 = k-th and (k+1)-th logits within 1e-5, bit 2 = two
                 // adjacent chosen logits are
};

// row: the token's E raw logits (global or shared memory); bias: [E] or nullptr.
// Lane l holds experts l, l + 32, ... (NV = ceil(E / 32) of them, NV a power of two
// <= kWarpTopkVals), sorted once by (value descending, expert ascending) with a small
// sorting network.  Then k + 1 rounds (the extra round finds the (k+1)-th value for
// the near-tie flag) each take the warp-wide largest head -- equal values to the lower
// expert -- with two warp reductions, and the winning lane drops its head.  Requires
// 1 <= k <= 32 and E <= 32 * NV.
template <int NV>
__device__ __forceinline__ WarpTopk warp_topk_nv(const float* row, const float* bias, int E, int k,
                                                 int normalize, int lane) {
    float v[NV];
    uint32_t key[NV];
    int id[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int e = lane + 32 * i;
        float x = -INFINITY;
        if (e < E) {
            x = row[e];
            if (bias) x += bias[e];
        }
        v[i] = x;
        key[i] = e < E ? order_key(x) : 0u;   // 0: below every real value
        id[i] = e < E ? e : 0x7fffffff;
    }
    // odd-even transposition sort of the lane's NV entries (NV <= 8)
#pragma unroll
    for (int pass = 0; pass < NV; ++pass) {
#pragma unroll
        for (int i = pass & 1; i + 1 < NV; i += 2) {
            const bool swap = key[i + 1] > key[i] || (key[i + 1] == key[i] && id[i + 1] < id[i]);
            const uint32_t k0 = key[i], k1 = key[i + 1];
            const int i0 = id[i], i1 = id[i + 1];
            key[i] = swap ? k1 : k0;
            key[i + 1] = swap ? k0 : k1;
            id[i] = swap ? i1 : i0;
            id[i + 1] = swap ? i0 : i1;
        }
    }
    const int rounds = min(k + 1, E);
    float sel_v = -INFINITY, next_v = -INFINITY;
    int sel_i = -1;
#pragma unroll 1
    for (int r = 0; r < rounds; ++r) {
        const uint32_t m = __reduce_max_sync(0xffffffffu, key[0]);
        const int wi = static_cast<int>(
            __reduce_min_sync(0xffffffffu, static_cast<uint32_t>(key[0] == m ? id[0] : 0x7fffffff)));
        if (wi == id[0]) {   // this lane's head was taken: the next entry moves up
#pragma unroll
            for (int i = 0; i + 1 < NV; ++i) {
                key[i] = key[i + 1];
                id[i] = id[i + 1];
            }
            key[NV - 1] = 0u;
            id[NV - 1] = 0x7fffffff;
        }
        const float wv = key_value(m);
        if (r == lane) {
            sel_v = wv;
            sel_i = wi;
        }
        if (r == k) next_v = wv;
    }
    const float vmax = __shfl_sync(0xffffffffu, sel_v, 0);
    const float num = (lane < k) ? expf(sel_v - vmax) : 0.f;
    float part = num;
    if (!normalize) {
        part = 0.f;
#pragma unroll
        for (int i = 0; i < NV; ++i)
            if (lane + 32 * i < E) part += expf(v[i] - vmax);
    }
    const float den = warp_sum(part);
    const float prev_v = __shfl_down_sync(0xffffffffu, sel_v, 1);
    const bool within = lane + 1 < k && (sel_v - prev_v) < kNearTieGap;
    const float kth = __shfl_sync(0xffffffffu, sel_v, k - 1);
    const unsigned wb = __ballot_sync(0xffffffffu, within);
    WarpTopk res;
    res.idx = sel_i;
    res.w = num / den;
    res.flags = ((k < E && kth - next_v < kNearTieGap) ? 1 : 0) | (wb ? 2 : 0);
    return res;
}

__device__ __forceinline__ WarpTopk warp_topk(const float* row, const float* bias, int E, int k,
                                              int normalize, int lane) {
    if (E <= 32) return warp_topk_nv<1>(row, bias, E, k, normalize, lane);
    if (E <= 64) return warp_topk_nv<2>(row, bias, E, k, normalize, lane);
    if (E <= 128) return warp_topk_nv<4>(row, bias, E, k, normalize, lane);
    return warp_topk_nv<8>(row, bias, E, k, normalize, lane);
}

}  // namespace moe
