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

__device__ __forceinline__ uint4 combine_vec_bf16(const uint4* __restrict__ y, int nvec,
                                                  const int32_t* __restrict__ perm_dst,
                                                  const float* __restrict__ topk_w, int t, int k,
                                                  int v, int rows_max) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int j0 = 0; j0 < k; j0 += kCombineUnroll) {
        float f[kCombineUnroll][8];
        float w[kCombineUnroll];
#pragma unroll
        for (int jj = 0; jj < kCombineUnroll; ++jj) {
            const int j = j0 + jj;
            int r = -1;
            w[jj] = 0.f;
            if (j < k) {
                r = perm_dst[static_cast<size_t>(t) * k + j];
                w[jj] = topk_w[static_cast<size_t>(t) * k + j];
            }
            if (r < 0 || r >= rows_max) {
                w[jj] = 0.f;
#pragma unroll
                for (int i = 0; i < 8; ++i) f[jj][i] = 0.f;
            } else {
                unpack_bf16x8(y[static_cast<size_t>(r) * nvec + v], f[jj]);
            }
        }
#pragma unroll
        for (int jj = 0; jj < kCombineUnroll; ++jj)
            if (j0 + jj < k) {
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] = fmaf(w[jj], f[jj][i], acc[i]);
            }
    }
    return pack_bf16x8(acc);
}

}  // namespace moe
