// Weighted combine (un-permute) and the fc1 layout conversion.
//
// Combine: out[t] = sum_j topk_w[t, j] * y_perm[perm_dst[t*k + j]] in float32, slot
// order j = 0..k-1, no atomics, so the result is bitwise reproducible; stored in the
// input dtype (the CastLike around the fused op, "Gemma 4 MoE: re-enable fused
// com.microsoft::MoE op - #326", "Changes").
//
// Convert: "Weight layout" of the same page -- Hugging Face's gate_up_proj is
// chunked [E, 2I, H] (gate rows first, then up rows); the interleaved layout of
// swiglu_fusion = 1 is the Reshape [E,2,I,H] -> Transpose [E,I,2,H] -> Reshape
// [E,2I,H], i.e. dst row 2j+s of expert e is src row s*I+j.
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

template <bool BF16>
__global__ void combine_kernel(const void* __restrict__ y_perm, const int32_t* __restrict__ perm_dst,
                               const float* __restrict__ topk_w, int T, int H, int k,
                               int rows_max, void* __restrict__ out) {
    __shared__ int s_row[kMaxExperts];
    __shared__ float s_w[kMaxExperts];
    constexpr int VEC = BF16 ? 8 : 4;
    const int nvec = H / VEC;
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        __syncthreads();
        for (int j = threadIdx.x; j < k; j += blockDim.x) {
            const int r = perm_dst[static_cast<size_t>(t) * k + j];
            s_row[j] = (r >= 0 && r < rows_max) ? r : -1;
            s_w[j] = topk_w[static_cast<size_t>(t) * k + j];
        }
        __syncthreads();
        for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
            float acc[VEC];
#pragma unroll
            for (int i = 0; i < VEC; ++i) acc[i] = 0.f;
            for (int j = 0; j < k; ++j) {
                const int r = s_row[j];
                if (r < 0) continue;
                const float w = s_w[j];
                float f[VEC];
                if constexpr (BF16) {
                    unpack_bf16x8(__ldg(reinterpret_cast<const uint4*>(y_perm) +
                                        static_cast<size_t>(r) * nvec + v),
                                  f);
                } else {
                    const float4 q = __ldg(reinterpret_cast<const float4*>(y_perm) +
                                           static_cast<size_t>(r) * nvec + v);
                    f[0] = q.x; f[1] = q.y; f[2] = q.z; f[3] = q.w;
                }
#pragma unroll
                for (int i = 0; i < VEC; ++i) acc[i] = fmaf(w, f[i], acc[i]);
            }
            if constexpr (BF16) {
                reinterpret_cast<uint4*>(out)[static_cast<size_t>(t) * nvec + v] = pack_bf16x8(acc);
            } else {
                reinterpret_cast<float4*>(out)[static_cast<size_t>(t) * nvec + v] =
                    make_float4(acc[0], acc[1], acc[2], acc[3]);
            }
        }
    }
}

__global__ void __launch_bounds__(256)
convert_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int E, int I,
               int vec_per_row) {
    const int lane = threadIdx.x & 31;
    const long long rows = static_cast<long long>(E) * 2 * I;
    const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
    for (long long d = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
         d < rows; d += warps) {
        const long long e = d / (2 * I);
        const int r = static_cast<int>(d - e * 2 * I);
        const int j = r >> 1, s = r & 1;
        const long long srow = e * 2 * I + static_cast<long long>(s) * I + j;
        const uint4* a = src + srow * vec_per_row;
        uint4* b = dst + d * vec_per_row;
        for (int v = lane; v < vec_per_row; v += 32) b[v] = __ldg(a + v);
    }
}

}  // namespace

cudaError_t launch_combine(const void* y_perm, const int32_t* perm_dst, const float* topk_w,
                           int T, int H, int k, bool bf16, void* out, cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    const int nvec = H / (bf16 ? 8 : 4);
    int threads = ((nvec + 31) / 32) * 32;
    if (threads > 512) threads = 512;
    if (threads < 64) threads = 64;
    int blocks = T;
    const int cap = device_sm_count() * 16;
    if (blocks > cap) blocks = cap;
    const int rows_max = T * k;
    if (bf16)
        combine_kernel<true><<<blocks, threads, 0, s>>>(y_perm, perm_dst, topk_w, T, H, k, rows_max,
                                                        out);
    else
        combine_kernel<false><<<blocks, threads, 0, s>>>(y_perm, perm_dst, topk_w, T, H, k,
                                                         rows_max, out);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_convert(const void* src, void* dst, int E, int I, int H, int elem_bytes,
                           cudaStream_t s) {
    const long long rows = static_cast<long long>(E) * 2 * I;
    if (rows <= 0) return cudaSuccess;
    const int vec = H * elem_bytes / 16;
    long long blocks = (rows + 7) / 8;
    const long long cap = static_cast<long long>(device_sm_count()) * 16;
    if (blocks > cap) blocks = cap;
    convert_kernel<<<static_cast<int>(blocks), 256, 0, s>>>(static_cast<const uint4*>(src),
                                                             static_cast<uint4*>(dst), E, I, vec);
    count_launch();
    return cudaGetLastError();
}

}  // namespace moe
