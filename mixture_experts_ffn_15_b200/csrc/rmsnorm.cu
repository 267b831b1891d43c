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
// A row is spread over TPR threads (TPR = 32 .. 256, so that a thread holds at most a
// few 16-byte vectors of it): every thread issues all its loads before it uses any,
// the float64 partial sums of squares (every float32 square is exact in float64) are
// reduced over the row's threads in a fixed order, then each thread scales, multiplies
// by the weight and stores its vectors (re-read from L1).  The same launch may clear a
// range of the layer's workspace, so that the normalised layer needs no extra launch.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kNormThreads = 256;
constexpr int kNormBatch = 2;   // vectors per thread loaded before any is used

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
__device__ __forceinline__ void load_vec(const uint4& q, float* f) {
    if constexpr (BF16) {
        unpack_bf16x8(q, f);
    } else {
        f[0] = __uint_as_float(q.x);
        f[1] = __uint_as_float(q.y);
        f[2] = __uint_as_float(q.z);
        f[3] = __uint_as_float(q.w);
    }
}

// y = round((x r) w) for one 16-byte vector
template <bool BF16>
__device__ __forceinline__ uint4 norm_vec(const uint4& q, const uint4& g, double r) {
    float f[8], gw[8];
    load_vec<BF16>(q, f);
    load_vec<BF16>(g, gw);
    if constexpr (BF16) {
        uint32_t b[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            b[i] = bf16_bits_from_f64((static_cast<double>(f[i]) * r) * static_cast<double>(gw[i]));
        return make_uint4(b[0] | (b[1] << 16), b[2] | (b[3] << 16), b[4] | (b[5] << 16),
                          b[6] | (b[7] << 16));
    } else {
        float z[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            z[i] = __double2float_rn((static_cast<double>(f[i]) * r) * static_cast<double>(gw[i]));
        return make_uint4(__float_as_uint(z[0]), __float_as_uint(z[1]), __float_as_uint(z[2]),
                          __float_as_uint(z[3]));
    }
}

template <bool BF16, int TPR>
__global__ void __launch_bounds__(kNormThreads)
rmsnorm_kernel(const void* __restrict__ x, const void* __restrict__ w, int T, int H, double eps,
               void* __restrict__ y, uint4* __restrict__ clear, int n_clear) {
    constexpr int RPB = kNormThreads / TPR;   // rows per block
    constexpr int WPR = TPR / 32;             // warps per row
    constexpr int VEC = BF16 ? 8 : 4;
    __shared__ double s_part[kNormThreads / 32];
    pdl_wait();
    pdl_trigger();
    for (int i = blockIdx.x * kNormThreads + threadIdx.x; i < n_clear; i += gridDim.x * kNormThreads)
        clear[i] = make_uint4(0u, 0u, 0u, 0u);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slot = threadIdx.x / TPR, j = threadIdx.x % TPR;
    const int nv = H / VEC;
    const uint4* wv = reinterpret_cast<const uint4*>(w);
    // the row loop is uniform over the block (the reduction below synchronises it)
    for (int t0 = blockIdx.x * RPB; t0 < T; t0 += gridDim.x * RPB) {
        const int t = t0 + slot;
        const bool live = t < T;
        const uint4* xr = reinterpret_cast<const uint4*>(x) + static_cast<size_t>(live ? t : 0) * nv;
        double ss = 0.0;
        if (live) {
            for (int base = j; base < nv; base += TPR * kNormBatch) {
                uint4 q[kNormBatch];
#pragma unroll
                for (int b = 0; b < kNormBatch; ++b) {
                    const int v = base + b * TPR;
                    q[b] = v < nv ? __ldg(xr + v) : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int b = 0; b < kNormBatch; ++b) {
                    float f[8];
                    load_vec<BF16>(q[b], f);
#pragma unroll
                    for (int i = 0; i < VEC; ++i)
                        ss = fma(static_cast<double>(f[i]), static_cast<double>(f[i]), ss);
                }
            }
        }
        ss = warp_sum_f64(ss);
        if constexpr (WPR > 1) {
            if (lane == 0) s_part[warp] = ss;
            __syncthreads();
            ss = 0.0;
#pragma unroll
            for (int i = 0; i < WPR; ++i) ss += s_part[slot * WPR + i];
            __syncthreads();   // s_part is written again by the next row
        }
        if (!live) continue;
        const double r = 1.0 / sqrt(ss / static_cast<double>(H) + eps);
        uint4* yr = reinterpret_cast<uint4*>(y) + static_cast<size_t>(t) * nv;
        for (int base = j; base < nv; base += TPR * kNormBatch) {
            uint4 q[kNormBatch], g[kNormBatch];
#pragma unroll
            for (int b = 0; b < kNormBatch; ++b) {
                const int v = base + b * TPR;
                if (v < nv) {
                    q[b] = __ldg(xr + v);
                    g[b] = __ldg(wv + v);
                }
            }
#pragma unroll
            for (int b = 0; b < kNormBatch; ++b) {
                const int v = base + b * TPR;
                if (v < nv) yr[v] = norm_vec<BF16>(q[b], g[b], r);
            }
        }
    }
}

template <bool BF16>
cudaError_t launch_norm_t(int tpr, dim3 grid, cudaStream_t s, const void* x, const void* w, int T,
                          int H, double eps, void* y, uint4* clear, int n_clear) {
    const dim3 block(kNormThreads);
    switch (tpr) {
        case 32: return launch_k(rmsnorm_kernel<BF16, 32>, grid, block, 0, s, x, w, T, H, eps, y, clear, n_clear);
        case 64: return launch_k(rmsnorm_kernel<BF16, 64>, grid, block, 0, s, x, w, T, H, eps, y, clear, n_clear);
        case 128: return launch_k(rmsnorm_kernel<BF16, 128>, grid, block, 0, s, x, w, T, H, eps, y, clear, n_clear);
        default: return launch_k(rmsnorm_kernel<BF16, 256>, grid, block, 0, s, x, w, T, H, eps, y, clear, n_clear);
    }
}

}  // namespace

cudaError_t launch_rmsnorm(const void* x, const void* w, int T, int H, float eps, bool bf16,
                           void* y, void* clear, size_t clear_bytes, cudaStream_t s) {
    if ((clear_bytes & 15) != 0 || (reinterpret_cast<uintptr_t>(clear) & 15) != 0)
        return cudaErrorInvalidValue;
    const long long n_clear = static_cast<long long>(clear_bytes / 16);
    // threads per row: the smallest of 32 .. 256 that leaves each thread at most two
    // vectors of the row (rows longer than 512 vectors take more batches)
    const int nv = H / (bf16 ? 8 : 4);
    int tpr = 32;
    while (tpr < kNormThreads && 2 * tpr < nv) tpr *= 2;
    const int rpb = kNormThreads / tpr;
    // one pass of the row loop per block: the hardware schedules the blocks in waves
    long long blocks = (static_cast<long long>(T) + rpb - 1) / rpb;
    const long long clear_blocks = (n_clear + 1023) / 1024;
    if (blocks < clear_blocks) blocks = clear_blocks;
    if (blocks > (1ll << 30)) blocks = 1ll << 30;
    if (blocks < 1) return cudaSuccess;
    const dim3 grid(static_cast<unsigned>(blocks));
    return bf16 ? launch_norm_t<true>(tpr, grid, s, x, w, T, H, static_cast<double>(eps), y,
                                      static_cast<uint4*>(clear), static_cast<int>(n_clear))
                : launch_norm_t<false>(tpr, grid, s, x, w, T, H, static_cast<double>(eps), y,
                                       static_cast<uint4*>(clear), static_cast<int>(n_clear));
}

}  // namespace moe
