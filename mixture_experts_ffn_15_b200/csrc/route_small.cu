// Routing for small batches (decode): router logits spread over many CTAs, then
// one CTA that does top-k, softmax, the bincount, the exclusive scan and the
// stable permutation without leaving shared memory.
//
// Same method as route.cu ("Gemma 4 MoE: re-enable fused com.microsoft::MoE op -
// #326", "Attribute set": k = top_k, normalize_routing_weights; "Contributing Gemma
// 4 support and ONNX export optimizations", "Key Technical Contributions": bincount
// of the chosen ids), shaped for T <= 512 tokens where a step is a few microseconds
// and every global-memory round trip shows.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "topk_warp.cuh"

namespace moe {
namespace {

// ---------------------------------------------------------------- router logits
// Block (expert group, token group): EPB experts x 16 tokens; the 256 threads split
// H in 16-byte vectors, each keeping EPB x 16 float32 partial dot products, reduced
// over the warp and then over the 8 warps in shared memory.  Block (0, 0) also
// clears the two header words of the layer's workspace (error word, counter).
constexpr int kSplitThreads = 256;
constexpr int kSplitTokens = 16;

template <bool BF16, int EPB>
__global__ void __launch_bounds__(kSplitThreads)
router_logits_split_kernel(const void* __restrict__ hidden, const void* __restrict__ router_w,
                           int T, int H, int E, float* __restrict__ logits,
                           int32_t* __restrict__ clear_words) {
    __shared__ float red[kSplitThreads / 32][EPB * kSplitTokens];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e0 = blockIdx.x * EPB;
    const int t0 = blockIdx.y * kSplitTokens;
    const int nt = min(kSplitTokens, T - t0);
    pdl_wait();
    pdl_trigger();
    if (clear_words && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x < 2)
        clear_words[threadIdx.x] = 0;
    float acc[EPB][kSplitTokens];
#pragma unroll
    for (int q = 0; q < EPB; ++q)
#pragma unroll
        for (int t = 0; t < kSplitTokens; ++t) acc[q][t] = 0.f;

    constexpr int VEC = BF16 ? 8 : 4;
    const int nv = H / VEC;
    for (int v = threadIdx.x; v < nv; v += kSplitThreads) {
        float wf[EPB][VEC];
#pragma unroll
        for (int q = 0; q < EPB; ++q) {
            const int e = min(e0 + q, E - 1);
            if constexpr (BF16) {
                unpack_bf16x8(__ldg(reinterpret_cast<const uint4*>(router_w) + static_cast<size_t>(e) * nv + v), wf[q]);
            } else {
                const float4 w4 = __ldg(reinterpret_cast<const float4*>(router_w) + static_cast<size_t>(e) * nv + v);
                wf[q][0] = w4.x; wf[q][1] = w4.y; wf[q][2] = w4.z; wf[q][3] = w4.w;
            }
        }
#pragma unroll
        for (int t = 0; t < kSplitTokens; ++t) {
            if (t < nt) {
                float xf[VEC];
                if constexpr (BF16) {
                    unpack_bf16x8(__ldg(reinterpret_cast<const uint4*>(hidden) + static_cast<size_t>(t0 + t) * nv + v), xf);
                } else {
                    const float4 x4 = __ldg(reinterpret_cast<const float4*>(hidden) + static_cast<size_t>(t0 + t) * nv + v);
                    xf[0] = x4.x; xf[1] = x4.y; xf[2] = x4.z; xf[3] = x4.w;
                }
#pragma unroll
                for (int q = 0; q < EPB; ++q)
#pragma unroll
                    for (int i = 0; i < VEC; ++i) acc[q][t] = fmaf(xf[i], wf[q][i], acc[q][t]);
            }
        }
    }
#pragma unroll
    for (int q = 0; q < EPB; ++q)
#pragma unroll
        for (int t = 0; t < kSplitTokens; ++t) {
            if (t < nt) {
                const float s = warp_sum(acc[q][t]);
                if (lane == 0) red[warp][q * kSplitTokens + t] = s;
            }
        }
    __syncthreads();
    if (threadIdx.x < EPB * kSplitTokens) {
        const int q = threadIdx.x / kSplitTokens, t = threadIdx.x % kSplitTokens;
        if (t < nt && e0 + q < E) {
            float s = 0.f;
#pragma unroll
            for (int w = 0; w < kSplitThreads / 32; ++w) s += red[w][threadIdx.x];
            logits[static_cast<size_t>(t0 + t) * E + e0 + q] = s;
        }
    }
}

// ---------------------------------------------------------------- single-CTA routing
constexpr int kSmallThreads = 1024;
constexpr int kSmallWarps = kSmallThreads / 32;
constexpr int kSmallMaskWords = kRouteSmallMaxT / 32;             // 16

__global__ void __launch_bounds__(kSmallThreads, 1) route_small_kernel(const RouteSmallArgs a) {
    __shared__ uint32_t s_mask[kMaxExperts * kSmallMaskWords];
    __shared__ int s_cnt[kMaxExperts];
    __shared__ int s_off[kMaxExperts + 1];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = a.T, E = a.E, k = a.k;
    const int words = (T + 31) / 32;
    pdl_wait();
    pdl_trigger();
    for (int i = threadIdx.x; i < E * words; i += kSmallThreads) s_mask[i] = 0;
    for (int e = threadIdx.x; e < E; e += kSmallThreads) s_cnt[e] = 0;
    for (int i = threadIdx.x; i < a.n_zero; i += kSmallThreads) a.zero_words[i] = 0;
    __syncthreads();

    // ---- top-k per token (one warp per token), weights, near-tie flags, bincount.
    // The token loop stays rolled: this kernel runs once per layer call with a cold
    // instruction cache, and unrolled copies of the body cost more to fetch than to run.
#pragma unroll 1
    for (int t = warp; t < T; t += kSmallWarps) {
        const WarpTopk r = warp_topk(a.logits + static_cast<size_t>(t) * E, a.bias, E, k,
                                     a.normalize, lane);
        if (lane < k) {
            a.topk_idx[static_cast<size_t>(t) * k + lane] = r.idx;
            a.topk_w[static_cast<size_t>(t) * k + lane] = r.w;
            if (static_cast<unsigned>(r.idx) < static_cast<unsigned>(E)) {
                atomicAdd(&s_cnt[r.idx], 1);
                atomicOr(&s_mask[r.idx * words + (t >> 5)], 1u << (t & 31));
            }
        }
        if (a.near_tie && lane == 0) a.near_tie[t] = r.flags;
    }
    __syncthreads();

    // ---- exclusive scan of the counts (warp 0)
    if (warp == 0) {
        constexpr int per = kMaxExperts / 32;   // compile-time: loc[] stays in registers
        int loc[per];
        int lsum = 0;
#pragma unroll
        for (int q = 0; q < per; ++q) {
            const int e = lane * per + q;
            loc[q] = e < E ? s_cnt[e] : 0;
            lsum += loc[q];
        }
        int incl = lsum;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d) incl += y;
        }
        int run = incl - lsum;
#pragma unroll
        for (int q = 0; q < per; ++q) {
            const int e = lane * per + q;
            if (e < E) {
                s_off[e] = run;
                a.offsets[e] = run;
                a.counts[e] = loc[q];
            }
            run += loc[q];
        }
        if (lane == 31) {
            s_off[E] = incl;
            a.offsets[E] = incl;
        }
    }
    __syncthreads();

    // ---- stable placement: rank of t among the tokens of its expert (the ids this
    // block wrote above are visible to it after the barrier)
#pragma unroll 1
    for (int t = warp; t < T; t += kSmallWarps) {
        if (lane < k) {
            const int e = a.topk_idx[static_cast<size_t>(t) * k + lane];
            int row = -1;
            if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) {
                const uint32_t* m = s_mask + e * words;
                const int w = t >> 5;
                int rank = __popc(m[w] & ((1u << (t & 31)) - 1u));
                for (int i = 0; i < w; ++i) rank += __popc(m[i]);
                row = s_off[e] + rank;
                a.perm_src[row] = t;
            }
            a.perm_dst[static_cast<size_t>(t) * k + lane] = row;
        }
    }
}

}  // namespace

cudaError_t launch_router_logits_split(const void* hidden, const void* router_w, int T, int H,
                                       int E, bool bf16, float* logits, int32_t* clear_words,
                                       cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    // four experts a block share every token vector they read; one expert a block when
    // four would leave most SMs idle (small batches: more, shorter blocks in flight, and
    // a kernel body a quarter the size, which a cold instruction cache fetches sooner).
    // The logits are the same bits either way: every sum runs in the same order.
    const long long tblocks = (T + kSplitTokens - 1) / kSplitTokens;
    const bool small = (E + 3) / 4 * tblocks < device_sm_count();
    const int epb = small ? 1 : 4;
    dim3 grid((E + epb - 1) / epb, (T + kSplitTokens - 1) / kSplitTokens);
    const dim3 block(kSplitThreads);
    if (bf16)
        return small ? launch_k(router_logits_split_kernel<true, 1>, grid, block, 0, s, hidden,
                                router_w, T, H, E, logits, clear_words)
                     : launch_k(router_logits_split_kernel<true, 4>, grid, block, 0, s, hidden,
                                router_w, T, H, E, logits, clear_words);
    return small ? launch_k(router_logits_split_kernel<false, 1>, grid, block, 0, s, hidden,
                            router_w, T, H, E, logits, clear_words)
                 : launch_k(router_logits_split_kernel<false, 4>, grid, block, 0, s, hidden,
                            router_w, T, H, E, logits, clear_words);
}

cudaError_t launch_route_small(const RouteSmallArgs& a, cudaStream_t s) {
    if (a.T <= 0) return cudaSuccess;
    return launch_k(route_small_kernel, dim3(1), dim3(kSmallThreads), 0, s, a);
}

}  // namespace moe
