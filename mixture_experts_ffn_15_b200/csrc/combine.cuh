// The weighted combine of one 8-wide bf16 output vector, shared by the standalone
// combine kernel and the fused decode FFN so that both give the same bits:
//   out[t, 8v .. 8v+7] = sum_j topk_w[t, j] * y_perm[perm_dst[t*k + j], 8v .. 8v+7]
// summed in float32 in slot order j = 0..k-1 (the CastLike output dtype of the op,
// "Gemma 4 MoE: re-enable fused com.microsoft::MoE op - #326", "Changes").
// Pairs whose row is outside [0, rows_max) are skipped.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kCombineUnroll = 8;

// Rows j0 .. j0+KC-1 of token t (16-byte vector v of each): raw bf16 vectors and
// weights; a slot past k, or a row outside [0, rows_max), holds weight 0 and a zero
// vector (its fma then adds +0, as for any zero row).
template <int KC>
struct CombineChunk {
    uint4 y[KC];
    float w[KC];
};

template <int KC>
__device__ __forceinline__ void combine_load(CombineChunk<KC>& c, const uint4* __restrict__ y,
                                             int nvec, const int32_t* __restrict__ perm_dst,
                                             const float* __restrict__ topk_w, int t, int k, int j0,
                                             int v, int rows_max) {
#pragma unroll
    for (int jj = 0; jj < KC; ++jj) {
        const int j = j0 + jj;
        int r = -1;
        float w = 0.f;
        if (j < k) {
            r = perm_dst[static_cast<size_t>(t) * k + j];
            w = topk_w[static_cast<size_t>(t) * k + j];
        }
        if (r < 0 || r >= rows_max) {
            c.w[jj] = 0.f;
            c.y[jj] = make_uint4(0u, 0u, 0u, 0u);
        } else {
            c.w[jj] = w;
            c.y[jj] = y[static_cast<size_t>(r) * nvec + v];
        }
    }
}

// acc += w_j y_j for the chunk's slots j < k, in slot order.
template <int KC>
__device__ __forceinline__ void combine_accumulate(float* acc, const CombineChunk<KC>& c, int k, int j0) {
#pragma unroll
    for (int jj = 0; jj < KC; ++jj)
        if (j0 + jj < k) {
            float f[8];
            unpack_bf16x8(c.y[jj], f);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = fmaf(c.w[jj], f[i], acc[i]);
        }
}

// P tokens t0, t0 + step, ... at once (the loads of all of them are in flight
// together), chunks of KC rows; every token's sum runs over j = 0 .. k-1 in order,
// so the result does not depend on KC or P.
template <int KC, int P>
__device__ __forceinline__ void combine_vecs_bf16(const uint4* __restrict__ y, int nvec,
                                                  const int32_t* __restrict__ perm_dst,
                                                  const float* __restrict__ topk_w, int t0, int step,
                                                  int k, int v, int rows_max, uint4* o) {
    float acc[P][8];
#pragma unroll
    for (int p = 0; p < P; ++p)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[p][i] = 0.f;
    for (int j0 = 0; j0 < k; j0 += KC) {
        CombineChunk<KC> c[P];
#pragma unroll
        for (int p = 0; p < P; ++p)
            combine_load<KC>(c[p], y, nvec, perm_dst, topk_w, t0 + p * step, k, j0, v, rows_max);
#pragma unroll
        for (int p = 0; p < P; ++p) combine_accumulate<KC>(acc[p], c[p], k, j0);
    }
#pragma unroll
    for (int p = 0; p < P; ++p) o[p] = pack_bf16x8(acc[p]);
}

__device__ __forceinline__ uint4 combine_vec_bf16(const uint4* __restrict__ y, int nvec,
                                                  const int32_t* __restrict__ perm_dst,
                                                  const float* __restrict__ topk_w, int t, int k,
                                                  int v, int rows_max) {
    uint4 o;
    combine_vecs_bf16<kCombineUnroll, 1>(y, nvec, perm_dst, topk_w, t, 0, k, v, rows_max, &o);
    return o;
}

}  // namespace moe
