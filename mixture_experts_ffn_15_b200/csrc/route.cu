// Routing kernels of the fused MoE layer.
//
// "Gemma 4 MoE: re-enable fused com.microsoft::MoE op - #326", "Attribute set":
// k = top_k experts per token, normalize_routing_weights = 1.  The router logits are
// hidden @ router_w^T (+ bias); the chosen experts are the k largest logits in
// descending order with ties to the lower expert index; their weights are the
// softmax over all experts, renormalised over the chosen k (normalize = 1) or kept
// as they are (normalize = 0).
//
// "Contributing Gemma 4 support and ONNX export optimizations", "Key Technical
// Contributions": the per-expert token count is a bincount over the chosen ids.
// topk_hist_kernel computes it per 128-token tile; the scatter kernel turns the
// tile counts into totals, offsets and per-tile bases.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

// ---------------------------------------------------------------- router logits (SIMT)
// One warp per (expert, group of 8 tokens): the warp streams the expert's router
// row once with 16-byte loads and keeps 8 float32 dot products; lanes are reduced
// with a butterfly.  Used for float32 and for small token counts in bf16.
constexpr int kLogitWarps = 8;
constexpr int kLogitTokens = 8;

template <bool BF16>
__global__ void __launch_bounds__(kLogitWarps * 32)
router_logits_simt_kernel(const void* __restrict__ hidden, const void* __restrict__ router_w,
                          int T, int H, int E, float* __restrict__ logits) {
    pdl_wait();
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * kLogitWarps + warp;
    const int t0 = blockIdx.y * kLogitTokens;
    if (e >= E) return;
    const int nt = min(kLogitTokens, T - t0);
    float acc[kLogitTokens];
#pragma unroll
    for (int t = 0; t < kLogitTokens; ++t) acc[t] = 0.f;

    if constexpr (BF16) {
        const int nv = H / 8;
        const uint4* w4 = reinterpret_cast<const uint4*>(
            static_cast<const __nv_bfloat16*>(router_w) + static_cast<size_t>(e) * H);
        const uint4* x4 = reinterpret_cast<const uint4*>(
            static_cast<const __nv_bfloat16*>(hidden) + static_cast<size_t>(t0) * H);
        for (int v = lane; v < nv; v += 32) {
            float wf[8];
            unpack_bf16x8(__ldg(w4 + v), wf);
#pragma unroll
            for (int t = 0; t < kLogitTokens; ++t) {
                if (t < nt) {
                    float xf[8];
                    unpack_bf16x8(__ldg(x4 + static_cast<size_t>(t) * nv + v), xf);
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[t] = fmaf(xf[i], wf[i], acc[t]);
                }
            }
        }
    } else {
        const int nv = H / 4;
        const float4* w4 =
            reinterpret_cast<const float4*>(static_cast<const float*>(router_w) + static_cast<size_t>(e) * H);
        const float4* x4 =
            reinterpret_cast<const float4*>(static_cast<const float*>(hidden) + static_cast<size_t>(t0) * H);
        for (int v = lane; v < nv; v += 32) {
            const float4 w = __ldg(w4 + v);
#pragma unroll
            for (int t = 0; t < kLogitTokens; ++t) {
                if (t < nt) {
                    const float4 x = __ldg(x4 + static_cast<size_t>(t) * nv + v);
                    acc[t] = fmaf(x.x, w.x, acc[t]);
                    acc[t] = fmaf(x.y, w.y, acc[t]);
                    acc[t] = fmaf(x.z, w.z, acc[t]);
                    acc[t] = fmaf(x.w, w.w, acc[t]);
                }
            }
        }
    }
#pragma unroll
    for (int t = 0; t < kLogitTokens; ++t) {
        const float s = warp_sum(acc[t]);
        if (lane == 0 && t < nt) logits[static_cast<size_t>(t0 + t) * E + e] = s;
    }
}

// ---------------------------------------------------------------- top-k + bincount + scan
constexpr int kHistThreads = 512;
constexpr int kHistWarps = kHistThreads / 32;
constexpr int kLanesVals = kMaxExperts / 32;   // logits held per lane

__global__ void __launch_bounds__(kHistThreads) topk_hist_kernel(const TopkHistArgs a) {
    __shared__ float s_val[kHistWarps][kMaxExperts + 1];
    __shared__ int s_sel[kHistWarps][kMaxExperts + 1];
    __shared__ int s_cnt[kMaxExperts];
    pdl_wait();
    pdl_trigger();

    const int tile = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = a.E, k = a.k;
    const int t_begin = tile * kTileTokens;
    const int t_end = min(a.T, t_begin + kTileTokens);

    // ---- phase A: top-k selection and routing weights, one warp per token
    if (a.logits != nullptr) {
        const int rounds = min(k + 1, E);   // the (k+1)-th value is kept for the tie flag
        for (int t = t_begin + warp; t < t_end; t += kHistWarps) {
            float v[kLanesVals];
#pragma unroll
            for (int i = 0; i < kLanesVals; ++i) {
                const int e = lane + 32 * i;
                float x = -INFINITY;
                if (e < E) {
                    x = a.logits[static_cast<size_t>(t) * E + e];
                    if (a.bias) x += a.bias[e];
                    if (a.logits_biased) a.logits_biased[static_cast<size_t>(t) * E + e] = x;
                }
                v[i] = x;
            }
            uint32_t taken = 0;
            for (int r = 0; r < rounds; ++r) {
                float bv = -INFINITY;
                int bi = 0x7fffffff;
#pragma unroll
                for (int i = 0; i < kLanesVals; ++i) {
                    const int e = lane + 32 * i;
                    if (e < E && !((taken >> i) & 1u) && (v[i] > bv || (v[i] == bv && e < bi))) {
                        bv = v[i];
                        bi = e;
                    }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                    if (ov > bv || (ov == bv && oi < bi)) {
                        bv = ov;
                        bi = oi;
                    }
                }
                if (bi < E && (bi & 31) == lane) taken |= 1u << (bi >> 5);
                if (lane == 0) {
                    s_val[warp][r] = bv;
                    s_sel[warp][r] = bi;
                }
            }
            __syncwarp();
            const float vmax = s_val[warp][0];
            float part = 0.f;
            if (a.normalize) {
                for (int j = lane; j < k; j += 32) part += expf(s_val[warp][j] - vmax);
            } else {
#pragma unroll
                for (int i = 0; i < kLanesVals; ++i)
                    if (lane + 32 * i < E) part += expf(v[i] - vmax);
            }
            const float den = warp_sum(part);
            for (int j = lane; j < k; j += 32) {
                a.topk_idx[static_cast<size_t>(t) * k + j] = s_sel[warp][j];
                a.topk_w[static_cast<size_t>(t) * k + j] = expf(s_val[warp][j] - vmax) / den;
            }
            if (a.near_tie != nullptr && lane == 0) {
                int f = 0;
                if (k < E && s_val[warp][k - 1] - s_val[warp][k] < kNearTieGap) f |= 1;
                for (int j = 0; j + 1 < k; ++j)
                    if (s_val[warp][j] - s_val[warp][j + 1] < kNearTieGap) {
                        f |= 2;
                        break;
                    }
                a.near_tie[t] = f;
            }
            __syncwarp();
        }
    }
    if (a.tile_counts == nullptr) return;

    // ---- phase B: bincount of this tile's expert ids
    __syncthreads();   // this block's topk_idx writes are visible to the block
    for (int e = threadIdx.x; e < E; e += kHistThreads) s_cnt[e] = 0;
    __syncthreads();
    const int npairs = (t_end - t_begin) * k;
    const int32_t* ids = a.topk_idx + static_cast<size_t>(t_begin) * k;
    for (int p = threadIdx.x; p < npairs; p += kHistThreads) {
        const int e = ids[p];
        if (static_cast<unsigned>(e) < static_cast<unsigned>(E))
            atomicAdd(&s_cnt[e], 1);
        else
            atomicOr(a.err, kErrBadExpert);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kHistThreads)
        a.tile_counts[static_cast<size_t>(tile) * E + e] = s_cnt[e];
}

}  // namespace

cudaError_t launch_router_logits_simt(const void* hidden, const void* router_w, int T, int H,
                                      int E, bool bf16, float* logits, cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    dim3 grid((E + kLogitWarps - 1) / kLogitWarps, (T + kLogitTokens - 1) / kLogitTokens);
    return bf16 ? launch_k(router_logits_simt_kernel<true>, grid, dim3(kLogitWarps * 32), 0, s,
                           hidden, router_w, T, H, E, logits)
                : launch_k(router_logits_simt_kernel<false>, grid, dim3(kLogitWarps * 32), 0, s,
                           hidden, router_w, T, H, E, logits);
}

cudaError_t launch_topk_hist(const TopkHistArgs& a, cudaStream_t s) {
    if (a.T <= 0) return cudaSuccess;
    return launch_k(topk_hist_kernel, dim3(num_token_tiles(a.T)), dim3(kHistThreads), 0, s, a);
}

}  // namespace moe
