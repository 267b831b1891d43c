/*
 * moe_b200.h -- C ABI of the fused mixture-of-experts FFN layer on B200 (sm_100a).
 *
 * The layer is the com.microsoft::MoE operator with standard SwiGLU, as stated in
 * "Gemma 4 MoE: re-enable fused com.microsoft::MoE op - #326" (onnxruntime/mobius
 * pull request), description and "Attribute set": per token, pick the k experts
 * with the largest router logits, weight them by the softmax renormalised over the
 * chosen k (normalize_routing_weights = 1), run each chosen expert's FFN
 *     act = silu(x fc1_gate^T) * (x fc1_up^T),   y = act fc2^T
 * with fc1 in the interleaved gate/up layout (swiglu_fusion = 1), and sum the
 * weighted expert outputs.  The per-expert token count is the bincount of the chosen
 * expert ids that "Contributing Gemma 4 support and ONNX export optimizations"
 * (Hugging Face forum, "Key Technical Contributions") puts in front of the grouped
 * matmul of grouped_mm_experts_forward.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers are DEVICE pointers owned by the caller, unless a parameter says
 *   otherwise.  The library never allocates device memory and never frees any.
 * - Every tensor is dense and row-major.  Weights are [out, in] (y = x W^T).
 * - `dt` gives the storage type of activations AND weights (hidden, router_w, fc1,
 *   fc2, x_perm, act, y_perm, out): MOE_F32 or MOE_BF16 (the *_q8 entry points take
 *   int8 expert weights with float32 row scales and bf16 everything else).  Router logits, routing
 *   weights and the router bias are always float32; indices and counts int32.
 *   Accumulation is float32 in every kernel; the bf16 expert GEMMs run on the
 *   tcgen05 tensor cores, the float32 path on plain FMA (no TF32).
 * - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = legacy
 *   default stream).  No entry point synchronises except moe_get_error.
 * - Argument errors are detected on the host before anything is enqueued and are
 *   returned as MOE_ERR_INVALID_ARG; a valid shape without an implemented kernel
 *   returns MOE_ERR_UNSUPPORTED; a failed launch returns MOE_ERR_CUDA.  Errors that
 *   only the device can see (an expert id out of range in the staged API, a wait
 *   that ran out) set bits in a device error word (see moe_get_error); the kernels
 *   then skip the offending work and never trap.
 * - Pointers to tensors must be 16-byte aligned; H and I must be multiples of 8.
 *   The bf16 path also needs H and I to be multiples of 64 (tensor-core K tiles).
 *   E <= 256 and 1 <= k <= E.
 * - Non-finite inputs are not checked; they propagate.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,   /* bad pointer, size, alignment or workspace too small */
    MOE_ERR_UNSUPPORTED = 2,   /* valid request with no implemented kernel */
    MOE_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
    MOE_ERR_DEVICE = 4,        /* moe_get_error: the device error word reports bad data */
    MOE_ERR_TIMEOUT = 5        /* moe_get_error: a bounded device wait ran out */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/* SwiGLU attributes of the op ("Attribute set": activation_alpha, activation_beta,
 * swiglu_limit; the GPT-OSS values 1.702, 1.0, 7.0 are the page's "1.702 multiplier",
 * "+1 bias on the up branch" and clipping).  With g and u the pre-activation gate and
 * up values of one output:
 *   act = (clip(u, -limit, limit) + beta) * min(g, limit) * sigmoid(alpha * min(g, limit))
 * Standard SwiGLU {1.0f, 0.0f, INFINITY} is silu(g) * u.  alpha and beta must be
 * finite and limit > 0 (INFINITY: no clipping), else MOE_ERR_INVALID_ARG. */
typedef struct { float alpha, beta, limit; } moe_swiglu;

/* Row layout of fc1 [E, 2I, H] ("Weight layout" of the pull request: the op's
 * swiglu_fusion = 1 is the interleaved layout, which the ORT CPU kernel requires; the
 * CUDA kernel it names accepts either, and so does every kernel here, reading the
 * chunked layout in place with no conversion pass):
 *   MOE_FC1_INTERLEAVED  row 2i = gate_i, row 2i+1 = up_i
 *   MOE_FC1_CHUNKED      row i = gate_i, row I+i = up_i (Hugging Face gate_up_proj)
 * fc1_bias [E, 2I], when given, is in the same layout.  Any other value is
 * MOE_ERR_INVALID_ARG. */
typedef enum { MOE_FC1_INTERLEAVED = 0, MOE_FC1_CHUNKED = 1 } moe_fc1_layout;

/* Bits of the device error word. */
#define MOE_DEVERR_BAD_EXPERT 1   /* an expert id outside [0, E) was skipped */
#define MOE_DEVERR_TIMEOUT    2   /* a bounded wait inside a kernel gave up */

/* ------------------------------------------------------------------ workspace sizes */

/* Bytes of device workspace that moe_forward needs for these sizes (pure host
 * arithmetic, no CUDA call).  Returns 0 for invalid sizes. */
size_t moe_workspace_size(int T, int H, int E, int k, int I, moe_dtype dt);

/* Bytes of scratch that moe_permute needs (the expert counts of every 128-token
 * tile).  Returns 0 for invalid sizes. */
size_t moe_permute_workspace_size(int T, int E);

/* Bytes of scratch that moe_expert_ffn needs (the activation rows [rows, I]). */
size_t moe_expert_ffn_workspace_size(int rows, int I, moe_dtype dt);

/* Pointer to the int32 device error word inside a moe_forward workspace (the
 * first 4 bytes).  moe_forward clears it at the start of every call. */
int32_t* moe_workspace_error_word(void* workspace);

/* ----------------------------------------------------------------------- staged API */

/* Router: logits, top-k selection and routing weights.
 * ("Attribute set": k = top_k, normalize_routing_weights.)
 *   hidden      [T, H]  dt
 *   router_w    [E, H]  dt
 *   router_bias [E] float32 or NULL; added to the logits before selection and softmax
 *   normalize   1: softmax over all E, keep the chosen k, divide by their sum;
 *               0: keep the chosen softmax probabilities as they are
 *   topk_idx    [T, k] int32 out: chosen experts, descending logit, ties to the
 *               lower expert index
 *   topk_w      [T, k] float32 out: routing weights in the same slot order
 *   logits      [T, E] float32 out (required): the logits the selection was made on
 *   near_tie    [T] int32 out or NULL: bit 1 = the k-th and (k+1)-th logits differ by
 *               less than 1e-5, bit 2 = two adjacent chosen logits do
 * T = 0 is a no-op. */
moe_status moe_route(const void* hidden, const void* router_w, const float* router_bias,
                     int T, int H, int E, int k, int normalize, moe_dtype dt,
                     int32_t* topk_idx, float* topk_w, float* logits, int32_t* near_tie,
                     void* stream);

/* Expert histogram (bincount), exclusive offsets and the stable permutation.
 * ("Contributing Gemma 4 support ...", "Key Technical Contributions": bincount.)
 *   topk_idx  [T, k] int32 in; ids outside [0, E) set MOE_DEVERR_BAD_EXPERT in
 *             *err_word and are left out of counts and rows
 *   counts    [E] int32 out; offsets [E+1] int32 out (offsets[E] = valid pairs)
 *   perm_src  [T*k] int32 out: permuted row r holds token perm_src[r]
 *   perm_dst  [T*k] int32 out: pair (t, j) lands in row perm_dst[t*k + j] (-1 if
 *             its id was out of range)
 *   Rows of one expert are contiguous, experts ascending, tokens ascending inside
 *   an expert (a stable permutation); the result is unique and deterministic.
 *   hidden    [T, H] dt in, x_perm [T*k, H] dt out: x_perm[r] = hidden[perm_src[r]];
 *             both may be NULL to skip the gather.
 *   err_word  int32 device word; bits are OR-ed in, never cleared here.
 *   workspace at least moe_permute_workspace_size(T, E) bytes, 256-byte aligned. */
moe_status moe_permute(const void* hidden, const int32_t* topk_idx, int T, int H, int E,
                       int k, moe_dtype dt, int32_t* counts, int32_t* offsets,
                       int32_t* perm_src, int32_t* perm_dst, void* x_perm,
                       int32_t* err_word, void* workspace, size_t ws_bytes, void* stream);

/* Grouped expert FFN over permuted rows.
 * ("Attribute set": SwiGLU attributes, interleaved fc1; grouped matmul of
 * grouped_mm_experts_forward.)
 *   x_perm   [rows, H] dt; rows offsets[e] .. offsets[e+1]-1 belong to expert e
 *   offsets  [E+1] int32 (device), non-decreasing, offsets[0] = 0, offsets[E] <= rows
 *   fc1      [E, 2I, H] dt in fc1_layout (interleaved: row 2i = gate_i, row 2i+1 = up_i;
 *            chunked: row i = gate_i, row I+i = up_i)
 *   fc2      [E, H, I] dt
 *   fc1_bias [E, 2I] dt (in fc1's layout) or NULL; fc2_bias [E, H] dt or
 *            NULL: the op's optional expert biases, added in float32 to the gate/up
 *            values before the activation and to the output
 *   y_perm   [rows, H] dt out: y_perm[r] = fc2_e act(g, u) + b2_e for r's expert e;
 *            rows at or beyond offsets[E] are not written
 *   workspace at least moe_expert_ffn_workspace_size(rows, I, dt) bytes. */
moe_status moe_expert_ffn(const void* x_perm, const int32_t* offsets, const void* fc1,
                          const void* fc2, const void* fc1_bias, const void* fc2_bias, int rows,
                          int H, int E, int I, moe_swiglu act, moe_fc1_layout fc1_layout,
                          moe_dtype dt, void* y_perm, void* workspace, size_t ws_bytes,
                          void* stream);

/* Weighted combine (un-permute).
 *   out[t, :] = sum_{j<k} topk_w[t, j] * y_perm[perm_dst[t*k + j], :], summed in
 *   float32 in slot order j = 0..k-1 (deterministic), stored as dt (the op's
 *   CastLike: "Changes" of the pull request).  Pairs with perm_dst < 0 are skipped. */
moe_status moe_combine(const void* y_perm, const int32_t* perm_dst, const float* topk_w,
                       int T, int H, int k, moe_dtype dt, void* out, void* stream);

/* ------------------------------------------------------------------------ the layer */

/* Pre-FFN RMSNorm, the step in front of the layer ("Contributing Gemma 4 support and
 * ONNX export optimizations", "Key Technical Contributions": Llama-style, the normed
 * states times the weight, not times 1 + weight):
 *   y[t, h] = (x[t, h] / sqrt(mean_h x[t, h]^2 + eps)) * weight[h]
 * evaluated in float64 and rounded once to dt (to nearest, ties to even), so the
 * result does not depend on the order of the sums.
 *   x [T, H] dt, weight [H] dt, y [T, H] dt (may not overlap x); eps finite and
 *   >= 0 (eps = 0 and an all-zero row give NaN, as the formula does).
 * T = 0 is a no-op. */
moe_status moe_rmsnorm(const void* x, const void* weight, int T, int H, float eps, moe_dtype dt,
                       void* y, void* stream);

/* The whole layer: [pre-FFN RMSNorm ->] route -> permute -> fc1 + SwiGLU -> fc2 ->
 * combine, all on `stream`, no host synchronisation.
 *   hidden [T, H], router_w [E, H], fc1 [E, 2I, H] in fc1_layout, fc2 [E, H, I]: dt
 *   norm_weight [H] dt or NULL: with a weight, `hidden` is the residual activation and
 *            the layer runs on moe_rmsnorm(hidden, norm_weight, norm_eps), which it
 *            computes into its workspace (the launch that clears the workspace header
 *            does it: no extra launch); NULL: hidden is the layer's input as is
 *   fc1_bias [E, 2I], fc2_bias [E, H] dt or NULL (as in moe_expert_ffn)
 *   router_bias [E] float32 or NULL; out [T, H] dt
 *   workspace >= moe_workspace_size(T, H, E, k, I, dt) bytes, 256-byte aligned; it
 *   holds every intermediate, and its first word is the device error word.
 * T = 0 is a no-op returning MOE_OK. */
moe_status moe_forward(const void* hidden, const void* norm_weight, float norm_eps,
                       const void* router_w, const float* router_bias,
                       const void* fc1, const void* fc2, const void* fc1_bias,
                       const void* fc2_bias, int T, int H, int E, int k, int I, int normalize,
                       moe_swiglu act, moe_fc1_layout fc1_layout, moe_dtype dt, void* out,
                       void* workspace, size_t ws_bytes, void* stream);

/* The whole layer without a workspace argument, for callers that cannot allocate
 * device memory while they run it (an engine plugin or a serving loop that forbids
 * allocation after start-up, a plain C host with no allocator of its own).  The
 * pages have no counterpart for this entry point.
 *   Arguments as moe_forward, minus workspace and ws_bytes.  The scratch is a fixed
 *   device array of MOE_STATIC_SCRATCH_BYTES inside the library, which every GPU
 *   that loads the library holds until the process exits.  Sizes whose
 *   moe_workspace_size(T, H, E, k, I, dt) exceeds MOE_STATIC_SCRATCH_BYTES (with
 *   E = 128, k = 8, H = 2816, I = 704 in bf16: up to 77 tokens) are rejected with
 *   MOE_ERR_INVALID_ARG before anything is enqueued; nothing is allocated, ever.
 *   The first call on a device looks up the array's device address (with that
 *   device current); make that first call before any stream capture.
 *   All calls share the array and it keeps the last call's contents (the parts
 *   that must start at zero are cleared by every call): calls whose work can
 *   overlap on the GPU, from two streams or two host threads, race on it. */
#define MOE_STATIC_SCRATCH_BYTES (8u << 20)
moe_status moe_forward_static(const void* hidden, const void* norm_weight, float norm_eps,
                              const void* router_w, const float* router_bias,
                              const void* fc1, const void* fc2, const void* fc1_bias,
                              const void* fc2_bias, int T, int H, int E, int k, int I,
                              int normalize, moe_swiglu act, moe_fc1_layout fc1_layout,
                              moe_dtype dt, void* out, void* stream);

/* ------------------------------------------------------------ int8 expert weights */

/* Weight-only int8 experts for decode-sized batches.  The pages name quantised MoE
 * (the QMoE operator of the CUDA pull request they cite) and 4-bit checkpoint weights
 * without a format; this library's reading: each weight row holds int8 values q in
 * [-127, 127] and one float32 scale, the weight being q * scale (symmetric, per output
 * row).  Activations, biases and outputs stay bf16; arithmetic as the bf16 path (q is
 * exact in bf16, the tensor cores accumulate sum_k q x in float32, the epilogue
 * multiplies by the row's scale before the bias and the activation).
 *   fc1_q [E, 2I, H] int8 in fc1_layout, fc1_scale [E, 2I] float32 (same layout)
 *   fc2_q [E, H, I] int8, fc2_scale [E, H] float32
 * Everything else as moe_forward / moe_expert_ffn with dt = MOE_BF16.  The int8
 * weights run in the decode FFN only: sizes where it does not apply (more than 64
 * routed rows per expert on average, H or 2I not multiples of 128) return
 * MOE_ERR_UNSUPPORTED.  Batches of at most 64 tokens run the whole layer in one
 * cooperative launch (bit 32 of moe_forward_path, as for bf16 weights); larger ones
 * route with the staged kernels first.  moe_workspace_size(T, H, E, k, I, MOE_BF16)
 * and moe_expert_ffn_workspace_size(rows, I, MOE_BF16) apply. */
moe_status moe_forward_q8(const void* hidden, const void* norm_weight, float norm_eps,
                          const void* router_w, const float* router_bias, const int8_t* fc1_q,
                          const float* fc1_scale, const int8_t* fc2_q, const float* fc2_scale,
                          const void* fc1_bias, const void* fc2_bias, int T, int H, int E, int k,
                          int I, int normalize, moe_swiglu act, moe_fc1_layout fc1_layout,
                          void* out, void* workspace, size_t ws_bytes, void* stream);
moe_status moe_expert_ffn_q8(const void* x_perm, const int32_t* offsets, const int8_t* fc1_q,
                             const float* fc1_scale, const int8_t* fc2_q, const float* fc2_scale,
                             const void* fc1_bias, const void* fc2_bias, int rows, int H, int E,
                             int I, moe_swiglu act, moe_fc1_layout fc1_layout, void* y_perm,
                             void* workspace, size_t ws_bytes, void* stream);

/* Layout conversion of fc1 from the Hugging Face chunked layout ("Weight layout":
 * [E, 2*inter, H], the first inter rows gate, the next inter rows up) to the
 * interleaved layout of swiglu_fusion = 1:  dst[e, 2j+s, :] = src[e, s*I + j, :].
 * This is the Reshape -> Transpose -> Reshape that the pull request folds into a
 * constant at session load.  src and dst must not overlap. */
moe_status convert_chunked_to_interleaved(const void* src, void* dst, int E, int I, int H,
                                          moe_dtype dt, void* stream);

/* ------------------------------------------------------------------------ errors */

/* Synchronises `stream`, reads the device error word and returns MOE_OK,
 * MOE_ERR_DEVICE (MOE_DEVERR_BAD_EXPERT set) or MOE_ERR_TIMEOUT.  If `bits` is not
 * NULL it receives the raw word (host pointer).  The word is not cleared. */
moe_status moe_get_error(const int32_t* err_word, void* stream, int32_t* bits);

/* A static, human-readable name of a status. */
const char* moe_status_string(moe_status s);

/* ------------------------------------------------------------------------ profiling */

/* Stage timing: when `events` is not NULL, moe_forward records the n_events (must
 * be 6) cudaEvent_t handles on its stream: before routing, after routing, after the
 * permutation, after fc1 + SwiGLU, after fc2, after the combine.  NULL turns the
 * recording off.  The handles stay owned by the caller.  Process-wide setting. */
moe_status moe_set_stage_events(void* const* events, int n_events);

/* Which kernels moe_forward runs for these sizes, as bits: 1 single-CTA routing
 * (T <= 512 and k <= 32), 2 fused decode FFN (fc1 + SwiGLU and fc2 in one launch,
 * weight rows on the MMA's M side), 4 tensor-core router, 8 token-row grouped GEMMs,
 * 16 float32 FMA FFN, 32 the routing inside the decode FFN's launch (the whole layer
 * in one cooperative launch, small bf16 batches).  0 for invalid sizes.  Pure host
 * arithmetic. */
int moe_forward_path(int T, int H, int E, int k, int I, moe_dtype dt);

/* Number of kernel launches the library has issued in this process (host-side count,
 * all devices).  A launch captured into a CUDA graph counts once, at capture. */
unsigned long long moe_kernel_launches(void);

/* Testing aid for the device-side failure detection, off by default: the next
 * moe_forward (or moe_forward_static) call that takes the one-launch path (bit 32 of
 * moe_forward_path) makes its routing grid barrier wait for one arrival more than its
 * grid provides, with a 1 ms limit instead of 2 s.  Every block then gives up before it
 * has issued any bulk copy or MMA, winds down, frees its tensor memory and sets
 * MOE_DEVERR_TIMEOUT in the call's error word (moe_get_error: MOE_ERR_TIMEOUT); the
 * call's outputs are not written.  One-shot: the setting is consumed by that call.
 * Process-wide; no counterpart on the pages. */
void moe_debug_arm_route_barrier_timeout(void);

/* Library version as major * 10000 + minor * 100 + patch. */
int moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
