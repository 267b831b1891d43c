// Pre-FFN RMSNorm, the step in front of the layer ("Contributing Gemma 4 support and
// ONNX export optimizations", "Key Technical Contributions": Gemma 4's norms are the
// Llama-style normed states times the weight, not times 1 + weight; the Rust
// weight-loader page lists the pre-FFN norm among each layer's four):
//   y[t, h] = round((x[t, h] / sqrt(mean_h x[t, h]^2 + eps)) * w[h])
// rounded ONCE to the storage dtype from a value within ~1e-14 relative of the exact
// one.  A rounding boundary is never that close in practice, so the layer's input does
// not depend on the order of the sums: the bits are those of the plain definition.
//
// bf16 rows stay in float32 arithmetic, whose conversions to and from float64 run at a
// small fraction of the float32 rate: the squares and the products x w of bf16 values
// are exact in float32; each vector's eight squares are summed with error-free
// transformations (TwoSum, D. Knuth, The Art of Computer Programming vol. 2, 4.2.2) and
// only the (sum, error) pair is widened into the float64 row sum; the scale r =
// 1 / sqrt(mean + eps) is taken in float64 once per row and split into r_hi + r_lo;
// t = fl(x w r_hi + fl(x w r_lo)) is within 0.51 float32 ulp of x w r, so rounding t
// to bf16 is right unless t lies within two float32 ulps of a bf16 midpoint (about 1e-4
// of the values); those take the exact path: x w r as an unevaluated float32 pair (the
// product's rounding error from an FMA, "TwoProd") rounded through round-to-odd
// (below).  float32 rows use float64 arithmetic directly.
//
// A row is spread over TPR threads (TPR = 32 .. 256, so that a thread holds at most
// kNormBatch 16-byte vectors of it): every thread issues all its loads before it uses
// any and keeps them in registers, the float64 partial sums of squares (every float32
// square is exact in float64) are reduced over the row's threads in a fixed order, then
// each thread scales its vectors, multiplies them by the weight and stores them.  Rows
// longer than 256 kNormBatch vectors take several batches (re-read for the second pass).  The same launch may clear a
// range of the layer's workspace, so that the normalised layer needs no extra launch.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kNormThreads = 256;
constexpr int kNormBatch = 6;   // vectors per thread loaded before any is used

// hi0 + lo0 (|lo0| at most a few float32 ulps of hi0; hi0 = 0 only if lo0 = 0) -> bf16
// with a single rounding to nearest, ties to even.  The pair is first renormalised with
// Fast2Sum (exact for |hi0| >= |lo0|; T. J. Dekker, "A floating-point technique for
// extending the available precision") into hi + lo, hi the float32 nearest to the sum
// and |lo| at most half an ulp of hi; then rounded to odd into float32 (24 >= 8 + 2 bits,
// so the second rounding cannot double-round; S. Boldo and G. Melquiond, "Emulation of
// FMA and correctly rounded sums: proved algorithms using rounding to odd") and from
// there to bf16, nearest even.  Round to odd: an inexact value goes to whichever of its
// two float32 neighbours has an odd last bit -- hi itself if odd, else hi's neighbour on
// lo's side.
__device__ __forceinline__ uint32_t bf16_bits_of_pair(float hi0, float lo0) {
    if (hi0 == 0.0f) return __float_as_uint(hi0) >> 16;   // a signed zero keeps its sign
    const float hi = __fadd_rn(hi0, lo0);
    const float lo = __fsub_rn(lo0, __fsub_rn(hi, hi0));
    uint32_t u = __float_as_uint(hi);
    if (lo != 0.0f && (u & 1u) == 0u) u = ((lo > 0.0f) == (hi > 0.0f)) ? u + 1u : u - 1u;
    return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(u))));
}

// a + b = s + e exactly (TwoSum).  The error-free transformations use the _rn
// intrinsics, which the compiler never contracts into an FMA or reorders.
__device__ __forceinline__ void two_sum(float a, float b, float& s, float& e) {
    s = __fadd_rn(a, b);
    const float bb = __fsub_rn(s, a);
    e = __fadd_rn(__fsub_rn(a, __fsub_rn(s, bb)), __fsub_rn(b, bb));
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

// y = round(x r w) for one 16-byte vector; r = r_hi + r_lo (bf16) or rd (float32)
template <bool BF16>
__device__ __forceinline__ uint4 norm_vec(const uint4& q, const uint4& g, float r_hi, float r_lo,
                                          double rd) {
    float f[8], gw[8];
    load_vec<BF16>(q, f);
    load_vec<BF16>(g, gw);
    if constexpr (BF16) {
        float t[8];
        bool near_mid = false;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float xw = __fmul_rn(f[i], gw[i]);       // exact: 8 x 8 significant bits
            // (a zero keeps its sign: -0 w r is -0, which the FMA's sum would lose)
            t[i] = xw == 0.0f ? __fmul_rn(xw, r_hi) : fmaf(xw, r_hi, __fmul_rn(xw, r_lo));
            const int low = static_cast<int>(__float_as_uint(t[i]) & 0xffffu);
            near_mid |= abs(low - 0x8000) <= 2;
        }
        if (!near_mid) return pack_bf16x8(t);
        uint32_t b[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float xw = __fmul_rn(f[i], gw[i]);
            const float p_hi = __fmul_rn(xw, r_hi);
            const float p_err = fmaf(xw, r_hi, -p_hi);      // the product's rounding error
            const float p_lo = fmaf(xw, r_lo, p_err);
            b[i] = bf16_bits_of_pair(p_hi, p_lo);
        }
        return make_uint4(b[0] | (b[1] << 16), b[2] | (b[3] << 16), b[4] | (b[5] << 16),
                          b[6] | (b[7] << 16));
    } else {
        float z[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            z[i] = __double2float_rn((static_cast<double>(f[i]) * rd) * static_cast<double>(gw[i]));
        return make_uint4(__float_as_uint(z[0]), __float_as_uint(z[1]), __float_as_uint(z[2]),
                          __float_as_uint(z[3]));
    }
}

// the sum of squares of one 16-byte vector, added to the float64 row sum
template <bool BF16>
__device__ __forceinline__ double add_squares(const uint4& q, double ss) {
    float f[8];
    load_vec<BF16>(q, f);
    if constexpr (BF16) {
        float hi = __fmul_rn(f[0], f[0]), lo = 0.0f;   // squares of bf16 values are exact
#pragma unroll
        for (int i = 1; i < 8; ++i) {
            float e;
            two_sum(hi, __fmul_rn(f[i], f[i]), hi, e);
            lo = __fadd_rn(lo, e);
        }
        return ss + (static_cast<double>(hi) + static_cast<double>(lo));
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) ss = fma(static_cast<double>(f[i]), static_cast<double>(f[i]), ss);
        return ss;
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
        uint4 q[kNormBatch];   // the thread's vectors of the row (first batch)
        if (live) {
            for (int base = j; base < nv; base += TPR * kNormBatch) {
#pragma unroll
                for (int b = 0; b < kNormBatch; ++b) {
                    const int v = base + b * TPR;
                    q[b] = v < nv ? __ldg(xr + v) : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int b = 0; b < kNormBatch; ++b) ss = add_squares<BF16>(q[b], ss);
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
        const float r_hi = static_cast<float>(r);
        const float r_lo = static_cast<float>(r - static_cast<double>(r_hi));
        uint4* yr = reinterpret_cast<uint4*>(y) + static_cast<size_t>(t) * nv;
        const bool one_batch = nv <= TPR * kNormBatch;   // q still holds the whole share
        for (int base = j; base < nv; base += TPR * kNormBatch) {
            uint4 g[kNormBatch];
#pragma unroll
            for (int b = 0; b < kNormBatch; ++b) {
                const int v = base + b * TPR;
                if (v < nv) {
                    if (!one_batch) q[b] = __ldg(xr + v);
                    g[b] = __ldg(wv + v);
                }
            }
#pragma unroll
            for (int b = 0; b < kNormBatch; ++b) {
                const int v = base + b * TPR;
                if (v < nv) yr[v] = norm_vec<BF16>(q[b], g[b], r_hi, r_lo, r);
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
    // threads per row: the smallest of 32 .. 256 that leaves each thread at most
    // kNormBatch vectors of the row (longer rows take more batches), widened while the
    // batch would not give every SM a block (small batches: spread each row out)
    const int nv = H / (bf16 ? 8 : 4);
    int tpr = 32;
    while (tpr < kNormThreads && kNormBatch * tpr < nv) tpr *= 2;
    while (tpr < kNormThreads && tpr < nv &&
           (static_cast<long long>(T) * tpr + kNormThreads - 1) / kNormThreads < device_sm_count())
        tpr *= 2;
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
