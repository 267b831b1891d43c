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
#include "combine.cuh"
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

// Block (token group, column slab): 128 threads, one 16-byte vector of the output row
// each; a block walks tokens t = blockIdx.x, blockIdx.x + gridDim.x, ...  The k rows of
// a token are loaded before they are summed (in slot order), so the loads overlap.  At
// most 64 registers a thread (8 blocks, 32 warps an SM): measured on 131072 rows of 4096
// (k = 4), 2 tokens x 4 rows in flight per thread at full occupancy ran at 6.25 TB/s,
// against 3.25 TB/s for 4 tokens x 4 rows at 127 registers (4 blocks an SM).
constexpr int kCombineThreads = 128;

template <bool BF16, int KC, int P>
__global__ void __launch_bounds__(kCombineThreads, 8)
combine_kernel(const void* __restrict__ y_perm, const int32_t* __restrict__ perm_dst,
               const float* __restrict__ topk_w, int T, int H, int k, int rows_max,
               void* __restrict__ out) {
    pdl_wait();
    pdl_trigger();
    constexpr int VEC = BF16 ? 8 : 4;
    const int nvec = H / VEC;
    const int v = blockIdx.y * kCombineThreads + threadIdx.x;
    if constexpr (BF16) {
        // P tokens per pass (about 16 row loads in flight per thread)
        if (v >= nvec) return;
        const uint4* y = reinterpret_cast<const uint4*>(y_perm);
        uint4* o = reinterpret_cast<uint4*>(out);
        const int step = gridDim.x;
        int t = blockIdx.x;
        for (; t + (P - 1) * step < T; t += P * step) {
            uint4 r[P];
            combine_vecs_bf16<KC, P>(y, nvec, perm_dst, topk_w, t, step, k, v, rows_max, r);
#pragma unroll
            for (int p = 0; p < P; ++p) o[static_cast<size_t>(t + p * step) * nvec + v] = r[p];
        }
        for (; t < T; t += step)
            o[static_cast<size_t>(t) * nvec + v] = combine_vec_bf16(y, nvec, perm_dst, topk_w, t, k, v, rows_max);
    } else {
        if (v >= nvec) return;
        for (int t = blockIdx.x; t < T; t += gridDim.x) {
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            for (int j = 0; j < k; ++j) {
                const int r = perm_dst[static_cast<size_t>(t) * k + j];
                if (r < 0 || r >= rows_max) continue;
                const float w = topk_w[static_cast<size_t>(t) * k + j];
                const float4 q = __ldg(reinterpret_cast<const float4*>(y_perm) + static_cast<size_t>(r) * nvec + v);
                acc[0] = fmaf(w, q.x, acc[0]);
                acc[1] = fmaf(w, q.y, acc[1]);
                acc[2] = fmaf(w, q.z, acc[2]);
                acc[3] = fmaf(w, q.w, acc[3]);
            }
            reinterpret_cast<float4*>(out)[static_cast<size_t>(t) * nvec + v] =
                make_float4(acc[0], acc[1], acc[2], acc[3]);
        }
    }
}

__global__ void __launch_bounds__(256)
convert_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int E, int I,
               int vec_per_row) {
    pdl_wait();
    pdl_trigger();
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

// words[0 .. n) = 0 with 16-byte stores (n a multiple of 4, words 16-byte aligned).
__global__ void __launch_bounds__(256) clear_kernel(uint4* __restrict__ words, int n4) {
    pdl_wait();
    pdl_trigger();
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += gridDim.x * blockDim.x)
        words[i] = make_uint4(0u, 0u, 0u, 0u);
}

}  // namespace

cudaError_t launch_clear(void* words, size_t bytes, cudaStream_t s) {
    if (bytes == 0) return cudaSuccess;
    if ((bytes & 15) != 0 || (reinterpret_cast<uintptr_t>(words) & 15) != 0) return cudaErrorInvalidValue;
    const long long n4 = static_cast<long long>(bytes / 16);
    long long blocks = (n4 + 1023) / 1024;
    if (blocks > device_sm_count()) blocks = device_sm_count();
    return launch_k(clear_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s,
                    static_cast<uint4*>(words), static_cast<int>(n4));
}

cudaError_t launch_combine(const void* y_perm, const int32_t* perm_dst, const float* topk_w,
                           int T, int H, int k, bool bf16, void* out, cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    const int nvec = H / (bf16 ? 8 : 4);
    const int slabs = (nvec + kCombineThreads - 1) / kCombineThreads;
    long long tok_blocks = (static_cast<long long>(device_sm_count()) * 16 + slabs - 1) / slabs;
    if (tok_blocks > T) tok_blocks = T;
    dim3 grid(static_cast<unsigned>(tok_blocks), static_cast<unsigned>(slabs));
    const int rows_max = T * k;
    if (!bf16)
        return launch_k(combine_kernel<false, 1, 1>, grid, dim3(kCombineThreads), 0, s, y_perm,
                        perm_dst, topk_w, T, H, k, rows_max, out);
    if (k <= 4)
        return launch_k(combine_kernel<true, 4, 2>, grid, dim3(kCombineThreads), 0, s, y_perm,
                        perm_dst, topk_w, T, H, k, rows_max, out);
    return launch_k(combine_kernel<true, 8, 1>, grid, dim3(kCombineThreads), 0, s, y_perm, perm_dst,
                    topk_w, T, H, k, rows_max, out);
}

cudaError_t launch_convert(const void* src, void* dst, int E, int I, int H, int elem_bytes,
                           cudaStream_t s) {
    const long long rows = static_cast<long long>(E) * 2 * I;
    if (rows <= 0) return cudaSuccess;
    const int vec = H * elem_bytes / 16;
    long long blocks = (rows + 7) / 8;
    const long long cap = static_cast<long long>(device_sm_count()) * 16;
    if (blocks > cap) blocks = cap;
    return launch_k(convert_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s,
                    static_cast<const uint4*>(src), static_cast<uint4*>(dst), E, I, vec);
}

}  // namespace moe
