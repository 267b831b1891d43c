// Pre-FFN RMSNorm, the step in front of the layer ("Contributing Gemma 4 support and
// ONNX export optimizations", "Key Technical Contributions": Gemma 4's norms are the
// Llama-style normed states times the weight, not times 1 + weight; the Rust
// weight-loader page lists the pre-FFN norm among each layer's four):
//   y[t, h] = round((x[t, h] / sqrt(mean_h x[t, h]^2 + eps)) * w[h])
// evaluated in float64 and rounded ONCE to the storage dtype.  The float64 value is
// within a few float64 ulps of the exact one and a bf16 rounding boundary is never
// that close in practice, so the layer's input does not depend on the order of the
// sums: the bits are those of the plain definition.
//
// One warp per row: a pass for the float64 sum of squares (every float32 square is
// exact in float64), then a pass that scales, multiplies by the weight and stores
// (the row is still in L1).  The same launch may clear a range of the layer's
// workspace, so that the normalised layer needs no extra launch.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kNormThreads = 256;
constexpr int kNormWarps = kNormThreads / 32;

// float64 -> bf16 with a single rounding to nearest, ties to even: round to odd into
// float32 first (24 >= 8 + 2 bits, so the second rounding cannot double-round; S. Boldo
// and G. Melquiond, "Emulation of FMA and correctly rounded sums: proved algorithms
// using rounding to odd"), then float32 -> bf16 to nearest even.
__device__ __forceinline__ uint32_t bf16_bits_from_f64(double y) {
    float f = __double2float_rz(y);
    if (static_cast<double>(f) != y) f = __uint_as_float(__float_as_uint(f) | 1u);
    return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(f)));
}

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <bool BF16>
__global__ void __launch_bounds__(kNormThreads)
rmsnorm_kernel(const void* __restrict__ x, const void* __restrict__ w, int T, int H, double eps,
               void* __restrict__ y, uint4* __restrict__ clear, int n_clear) {
    pdl_wait();
    pdl_trigger();
    for (int i = blockIdx.x * kNormThreads + threadIdx.x; i < n_clear; i += gridDim.x * kNormThreads)
        clear[i] = make_uint4(0u, 0u, 0u, 0u);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int VEC = BF16 ? 8 : 4;
    const int nv = H / VEC;
    const uint4* wv = reinterpret_cast<const uint4*>(w);
    for (int t = blockIdx.x * kNormWarps + warp; t < T; t += gridDim.x * kNormWarps) {
        const uint4* xr = reinterpret_cast<const uint4*>(x) + static_cast<size_t>(t) * nv;
        uint4* yr = reinterpret_cast<uint4*>(y) + static_cast<size_t>(t) * nv;
        double ss = 0.0;
        for (int v = lane; v < nv; v += 32) {
            const uint4 q = __ldg(xr + v);
            float f[8];
            if constexpr (BF16) unpack_bf16x8(q, f);
            else {
                f[0] = __uint_as_float(q.x); f[1] = __uint_as_float(q.y);
                f[2] = __uint_as_float(q.z); f[3] = __uint_as_float(q.w);
            }
#pragma unroll
            for (int i = 0; i < VEC; ++i) ss = fma(static_cast<double>(f[i]), static_cast<double>(f[i]), ss);
        }
        ss = warp_sum_f64(ss);
        const double r = 1.0 / sqrt(ss / static_cast<double>(H) + eps);
        for (int v = lane; v < nv; v += 32) {
            const uint4 q = __ldg(xr + v), g = __ldg(wv + v);
            float f[8], gw[8];
            uint4 o;
            if constexpr (BF16) {
                unpack_bf16x8(q, f);
                unpack_bf16x8(g, gw);
                uint32_t b[8];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    b[i] = bf16_bits_from_f64((static_cast<double>(f[i]) * r) * static_cast<double>(gw[i]));
                o = make_uint4(b[0] | (b[1] << 16), b[2] | (b[3] << 16), b[4] | (b[5] << 16),
                               b[6] | (b[7] << 16));
            } else {
                f[0] = __uint_as_float(q.x); f[1] = __uint_as_float(q.y);
                f[2] = __uint_as_float(q.z); f[3] = __uint_as_float(q.w);
                gw[0] = __uint_as_float(g.x); gw[1] = __uint_as_float(g.y);
                gw[2] = __uint_as_float(g.z); gw[3] = __uint_as_float(g.w);
                float z[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    z[i] = __double2float_rn((static_cast<double>(f[i]) * r) * static_cast<double>(gw[i]));
                o = make_uint4(__float_as_uint(z[0]), __float_as_uint(z[1]), __float_as_uint(z[2]),
                               __float_as_uint(z[3]));
            }
            yr[v] = o;
        }
    }
}

}  // namespace

cudaError_t launch_rmsnorm(const void* x, const void* w, int T, int H, float eps, bool bf16,
                           void* y, void* clear, size_t clear_bytes, cudaStream_t s) {
    if ((clear_bytes & 15) != 0 || (reinterpret_cast<uintptr_t>(clear) & 15) != 0)
        return cudaErrorInvalidValue;
    const long long n_clear = static_cast<long long>(clear_bytes / 16);
    long long blocks = (static_cast<long long>(T) + kNormWarps - 1) / kNormWarps;
    const long long cap = static_cast<long long>(device_sm_count()) * 8;
    if (blocks > cap) blocks = cap;
    const long long clear_blocks = (n_clear + 1023) / 1024;
    if (blocks < clear_blocks) blocks = clear_blocks < cap ? clear_blocks : cap;
    if (blocks < 1) return cudaSuccess;
    const auto kern = bf16 ? rmsnorm_kernel<true> : rmsnorm_kernel<false>;
    return launch_k(kern, dim3(static_cast<unsigned>(blocks)), dim3(kNormThreads), 0, s, x, w, T,
                    H, static_cast<double>(eps), y, static_cast<uint4*>(clear),
                    static_cast<int>(n_clear));
}

}  // namespace moe
