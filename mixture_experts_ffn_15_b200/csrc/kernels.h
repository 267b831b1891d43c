// Host-side launchers of the kernels (internal to the library, not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <utility>

#include "common.cuh"

namespace moe {

int device_sm_count();

// Records `ev` on `s`; inside a stream capture the record becomes an external
// event node, so that the event still times the replayed graph.
void record_event(cudaEvent_t ev, cudaStream_t s);

// Process-wide count of kernel launches issued by the library (host side).
void count_launch(int n = 1);

// Every kernel launch of the library: programmatic stream serialisation allowed, so
// the kernel may begin while its predecessor on the stream finishes (it waits with
// griddepcontrol.wait before touching memory), counted by count_launch().
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                     cudaStream_t s, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    count_launch();
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// The same launch, optionally cooperative: every block of the grid resident at once
// (a kernel with a grid-wide barrier); the launch fails rather than waits when they
// cannot all be resident.
template <typename... KArgs, typename... Args>
cudaError_t launch_k_coop(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t s, bool cooperative, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeCooperative;
    attr[1].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = cooperative ? 2 : 1;
    count_launch();
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------- rmsnorm.cu
// y [T, H] = the pre-FFN RMSNorm of x with weight w [H] (float64, one rounding to the
// dtype); the same launch zeroes `clear_bytes` (a multiple of 16) at `clear`.
cudaError_t launch_rmsnorm(const void* x, const void* w, int T, int H, float eps, bool bf16,
                           void* y, void* clear, size_t clear_bytes, cudaStream_t s);

// ---------------------------------------------------------------- route.cu
cudaError_t launch_router_logits_simt(const void* hidden, const void* router_w, int T, int H,
                                      int E, bool bf16, float* logits, cudaStream_t s);

struct TopkHistArgs {
    const float* logits = nullptr;   // [T, E] raw logits; nullptr: topk_idx is an input
    const float* bias = nullptr;     // [E] or nullptr
    float* logits_biased = nullptr;  // where to write logits + bias (nullptr: not written)
    int T = 0, E = 0, k = 0, normalize = 1;
    int32_t* topk_idx = nullptr;     // [T, k] out (or in when logits == nullptr)
    float* topk_w = nullptr;         // [T, k] out
    int32_t* near_tie = nullptr;     // [T] out or nullptr
    int32_t* tile_counts = nullptr;  // [ntiles, E] out (nullptr: no histogram)
    int32_t* err = nullptr;          // device error word
};
cudaError_t launch_topk_hist(const TopkHistArgs& a, cudaStream_t s);

inline int num_token_tiles(int T) { return (T + 127) / 128; }

// ---------------------------------------------------------------- route_small.cu
constexpr int kRouteSmallMaxT = 512;   // one CTA routes and permutes the whole batch
constexpr int kRouteSmallMaxK = 32;

cudaError_t launch_router_logits_split(const void* hidden, const void* router_w, int T, int H,
                                       int E, bool bf16, float* logits, int32_t* clear_words,
                                       cudaStream_t s);

struct RouteSmallArgs {
    const float* logits = nullptr;   // [T, E]
    const float* bias = nullptr;     // [E] or nullptr
    int T = 0, E = 0, k = 0, normalize = 1;
    int32_t* topk_idx = nullptr;     // [T, k]
    float* topk_w = nullptr;         // [T, k]
    int32_t* near_tie = nullptr;     // [T] or nullptr
    int32_t* counts = nullptr;       // [E]
    int32_t* offsets = nullptr;      // [E + 1]
    int32_t* perm_src = nullptr;     // [T * k]
    int32_t* perm_dst = nullptr;     // [T * k]
    int32_t* zero_words = nullptr;   // cleared by the kernel (the decode FFN's counters)
    int n_zero = 0;
};
cudaError_t launch_route_small(const RouteSmallArgs& a, cudaStream_t s);

// ---------------------------------------------------------------- permute.cu
// counts [E], offsets [E+1], perm_src, perm_dst from topk_idx and the per-tile counts
cudaError_t launch_scatter(const int32_t* topk_idx, const int32_t* tile_counts, int T, int E,
                           int k, int32_t* counts, int32_t* offsets, int32_t* perm_src,
                           int32_t* perm_dst, int32_t* err, cudaStream_t s);
cudaError_t launch_gather(const void* hidden, const int32_t* perm_src, const int32_t* offsets,
                          int E, int T, int rows_max, int H, int elem_bytes, void* x_perm,
                          cudaStream_t s);
// The same rows written token by token: x_perm[perm_dst[t k + j]] = hidden[t] (k <= 32;
// every row of hidden read once).
cudaError_t launch_gather_by_token(const void* hidden, const int32_t* perm_dst, int T, int k,
                                  int rows_max, int H, int elem_bytes, void* x_perm,
                                  cudaStream_t s);

// ---------------------------------------------------------------- combine.cu
// Zeroes `bytes` (a multiple of 16, 16-byte aligned) with a kernel, so that the launch
// overlaps the previous kernel on the stream (a memset node would not).
cudaError_t launch_clear(void* words, size_t bytes, cudaStream_t s);
cudaError_t launch_combine(const void* y_perm, const int32_t* perm_dst, const float* topk_w,
                           int T, int H, int k, bool bf16, void* out, cudaStream_t s);
cudaError_t launch_convert(const void* src, void* dst, int E, int I, int H, int elem_bytes,
                           cudaStream_t s);

// The op's attributes of the expert FFN: the SwiGLU attributes, the row layout of fc1
// and the optional expert biases (fc1_bias [E, 2I] in fc1's row layout, fc2_bias
// [E, H]; the activation dtype; nullptr = none).
//   fc1 interleaved: row 2i = gate_i, row 2i+1 = up_i;
//   fc1 chunked:     row i = gate_i,  row I+i  = up_i (the Hugging Face layout).
// Every kernel reads the chunked layout in place, as if it were interleaved: the
// bf16 kernels through a 4-D TMA view (H, gate/up, i, e) whose gate/up stride is one
// row for interleaved weights and I rows for chunked ones.
// Weight-only int8 experts (fc1_scale != nullptr): fc1 and fc2 hold int8 q and the
// weights are q * scale of their row (fc1_scale [E, 2I] in fc1's layout, fc2_scale
// [E, H], float32); the decode FFN kernel only.
struct FfnAttrs {
    SwigluAttr act{1.0f, 0.0f, INFINITY, 1};
    bool fc1_chunked = false;
    const void* fc1_bias = nullptr;
    const void* fc2_bias = nullptr;
    const float* fc1_scale = nullptr;
    const float* fc2_scale = nullptr;
    bool q8() const { return fc1_scale != nullptr; }
};

// Row of fc1 (or entry of fc1_bias) inside one expert that holds interleaved row j
// (gate_{j/2} for even j, up_{j/2} for odd j) in the given layout.
__host__ __device__ __forceinline__ int fc1_row(int j, int I, bool chunked) {
    return chunked ? (j & 1) * I + (j >> 1) : j;
}

// ---------------------------------------------------------------- ffn_simt.cu
cudaError_t launch_ffn_simt_f32(const float* x_perm, const int32_t* offsets, const float* fc1,
                                const float* fc2, int rows, int H, int E, int I, float* act,
                                float* y, cudaStream_t s, cudaEvent_t mid, const FfnAttrs& ep);

// ---------------------------------------------------------------- gemm_tc.cu
bool tc_ffn_supported(int H, int I);
// Router logits on the tensor cores with the routing in the epilogue: top-k, softmax
// weights, near-tie flags and the per-128-token-tile bincount (logits optional).
bool tc_route_supported(int H, int E, int k);
cudaError_t launch_route_tc(const void* hidden, const void* router_w, const float* bias, int T,
                            int H, int E, int k, int normalize, int32_t* topk_idx, float* topk_w,
                            int32_t* near_tie, float* logits, int32_t* tile_counts, int32_t* err,
                            cudaStream_t s);

// ---------------------------------------------------------------- gemm_pair.cu
// fc1 + SwiGLU and fc2 for large batches on CTA pairs (weight rows on M, M = 256 per
// pair): x_perm [rows, H] -> act [rows, I] -> y [rows, H]; `mid` (optional) is
// recorded between the two GEMMs.
bool pair_ffn_supported(int H, int I);
cudaError_t launch_ffn_pair(const void* x_perm, const int32_t* offsets, const void* fc1,
                            const void* fc2, int rows, int H, int E, int I, void* act, void* y,
                            int32_t* err, cudaStream_t s, cudaEvent_t mid, const FfnAttrs& ep);

// Decode FFN: fc1 + SwiGLU and fc2 in one persistent launch (weight rows on M).
bool decode_ffn_supported(int rows, int E, int H, int I);
int decode_ffn_counters(int rows, int E);   // int32 counters it needs, zero on entry
// tokens: `hidden` [T, H] gathered through perm_src, or x_perm [rows, H] if perm_src is null.
// With out != nullptr the launch also does the weighted combine into out [T, H].
// The same launch with the routing inside it (small batches): router logits on every
// CTA for its experts, a grid-wide barrier, then every CTA selects, counts and permutes
// the whole batch itself.  counters: decode_ffn_counters(T k, E) words, zero on entry.
constexpr int kFusedRouteMaxT = 64;
constexpr int kFusedRouteMaxRows = 512;
bool fused_route_supported(int T, int H, int E, int k, int I);
struct DecodeRoutedArgs {
    const void* hidden;        // [T, H] bf16
    const void* router_w;      // [E, H] bf16
    const float* bias;         // [E] or nullptr
    const void* fc1;           // [E, 2I, H] (int8 with ep.fc1_scale)
    const void* fc2;           // [E, H, I] (int8 with ep.fc2_scale)
    int T, H, E, k, I, normalize;
    float* logits;             // [T, E] scratch
    int32_t* topk_idx;         // [T, k] out
    float* topk_w;             // [T, k] out
    int32_t* near_tie;         // [T] out or nullptr
    int32_t* counts;           // [E] out
    int32_t* offsets;          // [E + 1] out
    int32_t* perm_src;         // [T k] out
    int32_t* perm_dst;         // [T k] out
    void* act;                 // [T k, I] scratch
    void* y;                   // [T k, H] scratch
    int32_t* counters;         // zero on entry
    int32_t* err;
    void* out;                 // [T, H]
    FfnAttrs ep;
};
cudaError_t launch_ffn_decode_routed(const DecodeRoutedArgs& a, cudaStream_t s);
// Testing aid: the next launch_ffn_decode_routed waits at its routing grid barrier for
// one arrival more than its grid provides, with a 1 ms limit (one-shot).
void arm_route_timeout_test();
bool take_route_timeout_test();

cudaError_t launch_ffn_decode(const void* tokens, const int32_t* perm_src, int T,
                              const int32_t* offsets, const void* fc1, const void* fc2, int rows,
                              int H, int E, int I, void* act, void* y, int32_t* done, int32_t* err,
                              const int32_t* perm_dst, const float* topk_w, int k, void* out,
                              cudaStream_t s, const FfnAttrs& ep);

}  // namespace moe
