// Device helpers shared by the kernels of the fused MoE layer.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

constexpr int kMaxExperts = 256;
constexpr int kErrBadExpert = 1;   // mirrors MOE_DEVERR_BAD_EXPERT
constexpr int kErrTimeout = 2;     // mirrors MOE_DEVERR_TIMEOUT
constexpr float kNearTieGap = 1e-5f;

// Token tile of the histogram / scatter kernels.
constexpr int kTileTokens = 128;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// 8 bf16 packed in 16 bytes -> 8 floats (exact).
__device__ __forceinline__ void unpack_bf16x8(const uint4& v, float* f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// Two floats -> packed bf16x2 (round to nearest even), low half = a.
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint4 pack_bf16x8(const float* f) {
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                      pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
}

// Programmatic dependent launch.  Every kernel of the library is launched so that it
// may start while the previous kernel on the stream is still running; pdl_wait()
// blocks until that kernel has completed and its memory is visible, so each kernel
// calls it before its first global-memory access.  pdl_trigger() lets the next
// kernel start its own prologue.  Both are no-ops for a plain launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// silu(g) * u in float32 (standard SwiGLU).
__device__ __forceinline__ float swiglu_f32(float g, float u) {
    return g / (1.0f + expf(-g)) * u;
}

// The same with the fast exponential and division intrinsics (a few ulp of float32,
// far below the bf16 rounding of the stored result); for large negative g the
// denominator overflows and the quotient is 0, as silu's limit.
__device__ __forceinline__ float swiglu_fast(float g, float u) {
    return __fdividef(g, 1.0f + __expf(-g)) * u;
}

// The op's SwiGLU attributes ("Gemma 4 MoE: re-enable fused com.microsoft::MoE op -
// #326", "Attribute set": activation_alpha, activation_beta, swiglu_limit):
//   act = (clip(u, -limit, limit) + beta) * g' * sigmoid(alpha * g'),  g' = min(g, limit)
// `standard` marks (1, 0, inf), which runs the plain silu(g) * u above.
struct SwigluAttr {
    float alpha, beta, limit;
    int standard;
};

__device__ __forceinline__ float swiglu_attr(float g, float u, const SwigluAttr& a) {
    if (a.standard) return swiglu_f32(g, u);
    if (a.limit < INFINITY) {
        g = fminf(g, a.limit);
        u = fminf(fmaxf(u, -a.limit), a.limit);
    }
    return g / (1.0f + expf(-a.alpha * g)) * (u + a.beta);
}

__device__ __forceinline__ float swiglu_attr_fast(float g, float u, const SwigluAttr& a) {
    if (a.standard) return swiglu_fast(g, u);
    if (a.limit < INFINITY) {
        g = fminf(g, a.limit);
        u = fminf(fmaxf(u, -a.limit), a.limit);
    }
    return __fdividef(g, 1.0f + __expf(-a.alpha * g)) * (u + a.beta);
}

__device__ __forceinline__ float bf16_at(const __nv_bfloat16* p, size_t i) {
    return __bfloat162float(p[i]);
}

}  // namespace moe
