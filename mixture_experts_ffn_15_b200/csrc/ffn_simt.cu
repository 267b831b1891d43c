// float32 grouped expert FFN on plain FMA (no TF32, which would not meet a 1e-4
// relative tolerance).  Same math as the tensor-core path:
//   act[r, i] = swiglu(x_perm[r] . gate_i + b1[gate_i], x_perm[r] . up_i + b1[up_i])
//   y[r, h]   = act[r] . fc2[e, h] + b2[e, h]
// for the rows r of expert e ("Gemma 4 MoE: re-enable fused com.microsoft::MoE op -
// #326", "Attribute set": SwiGLU attributes; the biases optional), gate_i and up_i the
// fc1 rows of either layout ("Weight layout": interleaved 2i / 2i+1, or chunked i / I+i).
#include "common.cuh"
#include "kernels.h"
#include "tile_map.cuh"

namespace moe {
namespace {

constexpr int SBM = 32, SBN = 64, SBK = 32;
static_assert(SBM * SBK % 256 == 0 && SBN * SBK % 256 == 0, "whole slices per thread");

// out[r, n] = A[r, :] . W[e, n, :] for the rows of each expert, 32 x 64 output tile
// per unit; with SWIGLU the adjacent (gate, up) columns are fused into one act value
// (column n of W is fc1's interleaved row n, read from the chunked layout in place when
// `chunked`).
template <bool SWIGLU>
__global__ void __launch_bounds__(256)
simt_grouped_gemm_kernel(const float* __restrict__ A, int lda, const float* __restrict__ W,
                         int n_w, int K, const int32_t* __restrict__ offsets, int E, int rows,
                         float* __restrict__ out, int ldo, const float* __restrict__ bias,
                         SwigluAttr act, bool chunked) {
    __shared__ float sA[SBM][SBK + 1];
    // W transposed, k-major: a thread's four output columns at one k are one 16-byte
    // load (rows padded to a multiple of 16 bytes)
    __shared__ __align__(16) float sW[SBK][SBN + 4];
    __shared__ int s_off[kMaxExperts + 1];
    __shared__ int s_pre[kMaxExperts + 1];
    const int tid = threadIdx.x;
    pdl_wait();
    pdl_trigger();
    // the tile map (offsets clamped to [0, rows] and made non-decreasing, tiles of SBM
    // rows per expert), built by one warp with all its loads in flight at once
    if (tid < 32) build_group_tiles(offsets, rows, nullptr, E, SBM, s_off, s_pre, tid);
    __syncthreads();
    const int NT = (n_w + SBN - 1) / SBN;
    const int total = s_pre[E] * NT;
    const int tx = tid & 15, ty = tid >> 4;
    for (int u = blockIdx.x; u < total; u += gridDim.x) {
        const int mt = u / NT, nt = u - (u / NT) * NT;
        int lo = 0, hi = E - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_pre[mid] <= mt) lo = mid; else hi = mid - 1;
        }
        const int e = lo;
        const int row0 = s_off[e] + (mt - s_pre[e]) * SBM;
        const int nrows = min(SBM, s_off[e + 1] - row0);
        const float* We = W + static_cast<size_t>(e) * n_w * K;
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        // the next K slice is loaded into registers while the current one is multiplied
        constexpr int kAPer = SBM * SBK / 256, kWPer = SBN * SBK / 256;
        float ra[kAPer], rw[kWPer];
        auto fetch = [&](int k0) {
#pragma unroll
            for (int j = 0; j < kAPer; ++j) {
                const int i = tid + j * 256, r = i / SBK, c = i - (i / SBK) * SBK;
                ra[j] = (r < nrows && k0 + c < K) ? A[static_cast<size_t>(row0 + r) * lda + k0 + c] : 0.f;
            }
#pragma unroll
            for (int j = 0; j < kWPer; ++j) {
                const int i = tid + j * 256, n = i / SBK, c = i - (i / SBK) * SBK;
                const int wn = nt * SBN + n;
                const int wr = SWIGLU ? fc1_row(wn, n_w / 2, chunked) : wn;
                rw[j] = (wn < n_w && k0 + c < K) ? We[static_cast<size_t>(wr) * K + k0 + c] : 0.f;
            }
        };
        fetch(0);
        for (int k0 = 0; k0 < K; k0 += SBK) {
#pragma unroll
            for (int j = 0; j < kAPer; ++j) {
                const int i = tid + j * 256;
                sA[i / SBK][i - (i / SBK) * SBK] = ra[j];
            }
#pragma unroll
            for (int j = 0; j < kWPer; ++j) {
                const int i = tid + j * 256;
                sW[i - (i / SBK) * SBK][i / SBK] = rw[j];
            }
            __syncthreads();
            if (k0 + SBK < K) fetch(k0 + SBK);
#pragma unroll 8
            for (int c = 0; c < SBK; ++c) {
                const float a0 = sA[ty * 2][c], a1 = sA[ty * 2 + 1][c];
                const float4 w4 = *reinterpret_cast<const float4*>(&sW[c][tx * 4]);
                const float w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    acc[0][q] = fmaf(a0, w[q], acc[0][q]);
                    acc[1][q] = fmaf(a1, w[q], acc[1][q]);
                }
            }
            __syncthreads();
        }
        const int n0 = nt * SBN + tx * 4;
        if (bias != nullptr) {   // the expert's bias of each output column
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int bn = SWIGLU ? fc1_row(n0 + q, n_w / 2, chunked) : n0 + q;
                const float b = n0 + q < n_w ? bias[static_cast<size_t>(e) * n_w + bn] : 0.f;
                acc[0][q] += b;
                acc[1][q] += b;
            }
        }
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            const int r = ty * 2 + rr;
            if (r >= nrows) continue;
            float* o = out + static_cast<size_t>(row0 + r) * ldo;
            if constexpr (SWIGLU) {
                if (n0 + 1 < n_w) o[n0 / 2] = swiglu_attr(acc[rr][0], acc[rr][1], act);
                if (n0 + 3 < n_w) o[n0 / 2 + 1] = swiglu_attr(acc[rr][2], acc[rr][3], act);
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (n0 + q < n_w) o[n0 + q] = acc[rr][q];
            }
        }
    }
}

int simt_grid(int rows, int E, int n_w) {
    const long long bound = (static_cast<long long>((rows + SBM - 1) / SBM) + E) * ((n_w + SBN - 1) / SBN);
    const long long cap = static_cast<long long>(device_sm_count()) * 8;
    return static_cast<int>(bound < cap ? bound : cap);
}

}  // namespace

cudaError_t launch_ffn_simt_f32(const float* x_perm, const int32_t* offsets, const float* fc1,
                                const float* fc2, int rows, int H, int E, int I, float* act,
                                float* y, cudaStream_t s, cudaEvent_t mid, const FfnAttrs& ep) {
    if (rows <= 0) return cudaSuccess;
    cudaError_t err = launch_k(simt_grouped_gemm_kernel<true>, dim3(simt_grid(rows, E, 2 * I)),
                               dim3(256), 0, s, x_perm, H, fc1, 2 * I, H, offsets, E, rows, act, I,
                               static_cast<const float*>(ep.fc1_bias), ep.act, ep.fc1_chunked);
    if (err != cudaSuccess) return err;
    if (mid) record_event(mid, s);
    return launch_k(simt_grouped_gemm_kernel<false>, dim3(simt_grid(rows, E, H)), dim3(256), 0, s,
                    static_cast<const float*>(act), I, fc2, H, I, offsets, E, rows, y, H,
                    static_cast<const float*>(ep.fc2_bias), ep.act, false);
}

}  // namespace moe
