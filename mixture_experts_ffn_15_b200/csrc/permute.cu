// Stable token permutation and row gather of the fused MoE layer.
//
// Pair (t, j) with expert e = topk_idx[t, j] goes to permuted row
//   offsets[e] + #{t' < t : some slot of t' chose e}
// i.e. the rows of an expert are contiguous and ordered by token (the grouped
// matmul of grouped_mm_experts_forward, "Contributing Gemma 4 support and ONNX
// export optimizations", "Key Technical Contributions"), and the offsets are the
// exclusive scan of the per-expert bincount.  The inputs are the per-128-token-tile
// expert counts; the result is unique and deterministic.
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kScatterThreads = 512;
constexpr int kMaskWords = kTileTokens / 32;

// One block per 128-token tile.  The block first turns the per-tile expert counts of
// ALL tiles (tile_counts [ntiles, E], a few KB from L2) into what it needs: the
// per-expert totals, their exclusive scan (the offsets; block 0 writes counts and
// offsets) and, for its own tile, the first row of every expert:
//   base[e] = offsets[e] + sum over earlier tiles of tile_counts[tile', e].
// Every block does this small reduction itself, so no block waits for another.
// Then the rank of a token among the tile's tokens of the same expert is a population
// count over a 128-bit membership mask.
__global__ void __launch_bounds__(kScatterThreads)
scatter_kernel(const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ tile_counts,
               int T, int E, int k, int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
               int32_t* __restrict__ perm_src, int32_t* __restrict__ perm_dst,
               int32_t* __restrict__ err) {
    __shared__ uint32_t s_mask[kMaxExperts * kMaskWords];
    __shared__ int s_tot[kScatterThreads];
    __shared__ int s_before[kScatterThreads];
    __shared__ int s_base[kMaxExperts];
    pdl_wait();
    pdl_trigger();
    const int tile = blockIdx.x;
    const int ntiles = gridDim.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t_begin = tile * kTileTokens;
    const int nt = min(kTileTokens, T - t_begin);
    for (int i = threadIdx.x; i < E * kMaskWords; i += kScatterThreads) s_mask[i] = 0;

    // ---- totals and earlier-tile sums per expert: thread (strip, e)
    const int strips = kScatterThreads / E;   // E <= 256: at least 2
    const int chunk = (ntiles + strips - 1) / strips;
    const int st = threadIdx.x / E, e_own = threadIdx.x - st * E;
    int tot = 0, before = 0;
    if (st < strips) {
        const int i0 = st * chunk, i1 = min(ntiles, i0 + chunk);
#pragma unroll 8
        for (int i = i0; i < i1; ++i) {
            const int c = tile_counts[static_cast<size_t>(i) * E + e_own];
            tot += c;
            before += (i < tile) ? c : 0;
        }
    }
    s_tot[threadIdx.x] = tot;
    s_before[threadIdx.x] = before;
    __syncthreads();
    if (warp == 0) {
        constexpr int per = kMaxExperts / 32;   // compile-time: loc[] stays in registers
        int loc[per];
        int lsum = 0;
#pragma unroll
        for (int q = 0; q < per; ++q) {
            const int e = lane * per + q;
            int t = 0;
            if (e < E)
                for (int ss = 0; ss < strips; ++ss) t += s_tot[ss * E + e];
            loc[q] = t;
            lsum += t;
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
                int b = run;
                for (int ss = 0; ss < strips; ++ss) b += s_before[ss * E + e];
                s_base[e] = b;
                if (tile == 0) {
                    offsets[e] = run;
                    counts[e] = loc[q];
                }
            }
            run += loc[q];
        }
        if (tile == 0 && lane == 31) offsets[E] = incl;
    }
    __syncthreads();

    // ---- membership masks, then ranks
    const int npairs = nt * k;
    const int32_t* ids = topk_idx + static_cast<size_t>(t_begin) * k;
    for (int p = threadIdx.x; p < npairs; p += kScatterThreads) {
        const int e = ids[p];
        const int tl = p / k;
        if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) {
            const uint32_t bit = 1u << (tl & 31);
            // the same expert twice in one token: reported, the ranks then collide
            if (atomicOr(&s_mask[e * kMaskWords + (tl >> 5)], bit) & bit) atomicOr(err, kErrBadExpert);
        }
    }
    __syncthreads();
    for (int p = threadIdx.x; p < npairs; p += kScatterThreads) {
        const int e = ids[p];
        const int tl = p / k;
        int32_t row = -1;
        if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) {
            const uint32_t* m = s_mask + e * kMaskWords;
            const int w = tl >> 5;
            int rank = __popc(m[w] & ((1u << (tl & 31)) - 1u));
            for (int q = 0; q < w; ++q) rank += __popc(m[q]);
            row = s_base[e] + rank;
            perm_src[row] = t_begin + tl;
        }
        perm_dst[static_cast<size_t>(t_begin) * k + p] = row;
    }
}

// x_perm[perm_dst[t k + j]] = hidden[t] for every pair (t, j); one warp per (token,
// chunk of chunk_vecs 16-byte vectors).  Walking the tokens (not the permuted rows)
// reads every row of hidden once, in order, and writes its k copies: by permuted row, a
// row would be read k times from far-apart places, i.e. from HBM each time once hidden
// exceeds L2.  Large batches take a whole row per warp; small ones split rows so that
// every SM gets warps.  Pairs whose row is outside [0, rows_max) (an id that was out of
// range) are skipped; rows that no pair names are not written.
__global__ void __launch_bounds__(256)
gather_by_token_kernel(const uint4* __restrict__ hidden, const int32_t* __restrict__ perm_dst,
                       int T, int k, int rows_max, int vec_per_row, int chunk_vecs,
                       uint4* __restrict__ x_perm) {
    pdl_wait();
    pdl_trigger();
    constexpr int kKMax = 32;
    const int lane = threadIdx.x & 31;
    const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
    const int nchunks = (vec_per_row + chunk_vecs - 1) / chunk_vecs;
    const long long items = static_cast<long long>(T) * nchunks;
    for (long long it = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
         it < items; it += warps) {
        const int t = static_cast<int>(it / nchunks);
        const int c = static_cast<int>(it - static_cast<long long>(t) * nchunks);
        // the token's destination rows: lane j holds row j (k <= 32)
        int dst = -1;
        if (lane < k) {
            const int r = perm_dst[static_cast<size_t>(t) * k + lane];
            dst = (r >= 0 && r < rows_max) ? r : -1;
        }
        const uint4* s = hidden + static_cast<size_t>(t) * vec_per_row;
        const int v_end = min(vec_per_row, (c + 1) * chunk_vecs);
        // 8 loads in flight per lane before the stores
        for (int v0 = c * chunk_vecs + lane; v0 < v_end; v0 += 32 * 8) {
            uint4 buf[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (v0 + 32 * q < v_end) buf[q] = __ldcs(s + v0 + 32 * q);
#pragma unroll 1
            for (int j = 0; j < k && j < kKMax; ++j) {
                const int r = __shfl_sync(0xffffffffu, dst, j);
                if (r < 0) continue;
                uint4* d = x_perm + static_cast<size_t>(r) * vec_per_row;
                // streaming stores: x_perm is read back once, by the grouped GEMM
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    if (v0 + 32 * q < v_end) __stcs(d + v0 + 32 * q, buf[q]);
            }
        }
    }
}

// x_perm[r] = hidden[perm_src[r]] for r < offsets[E]; one warp per row, 16-byte
// vectors.  A source index outside [0, T) (possible only after bad ids in the
// staged API) writes a zero row instead of reading out of bounds.
__global__ void __launch_bounds__(256)
gather_kernel(const uint4* __restrict__ hidden, const int32_t* __restrict__ perm_src,
              const int32_t* __restrict__ offsets, int E, int T, int rows_max, int vec_per_row,
              uint4* __restrict__ x_perm) {
    pdl_wait();
    pdl_trigger();
    const int rows = min(offsets[E], rows_max);
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (blockDim.x >> 5);
    for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
        const int src = perm_src[r];
        uint4* dst = x_perm + static_cast<size_t>(r) * vec_per_row;
        if (src < 0 || src >= T) {
            for (int v = lane; v < vec_per_row; v += 32) dst[v] = make_uint4(0, 0, 0, 0);
            continue;
        }
        // 8 loads in flight per lane before the stores
        const uint4* s = hidden + static_cast<size_t>(src) * vec_per_row;
        for (int v0 = lane; v0 < vec_per_row; v0 += 32 * 8) {
            uint4 buf[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (v0 + 32 * q < vec_per_row) buf[q] = __ldg(s + v0 + 32 * q);
            // streaming stores: x_perm is larger than L2 and read back from HBM anyway
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (v0 + 32 * q < vec_per_row) __stcs(dst + v0 + 32 * q, buf[q]);
        }
    }
}

}  // namespace

cudaError_t launch_scatter(const int32_t* topk_idx, const int32_t* tile_counts, int T, int E,
                           int k, int32_t* counts, int32_t* offsets, int32_t* perm_src,
                           int32_t* perm_dst, int32_t* err, cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    return launch_k(scatter_kernel, dim3(num_token_tiles(T)), dim3(kScatterThreads), 0, s, topk_idx,
                    tile_counts, T, E, k, counts, offsets, perm_src, perm_dst, err);
}

cudaError_t launch_gather_by_token(const void* hidden, const int32_t* perm_dst, int T, int k,
                                  int rows_max, int H, int elem_bytes, void* x_perm,
                                  cudaStream_t s) {
    if (T <= 0 || k > 32) return T <= 0 ? cudaSuccess : cudaErrorInvalidValue;
    const int vec = H * elem_bytes / 16;
    const int sms = device_sm_count();
    // batches of fewer than 16 tokens per SM split their rows into chunks (a multiple of
    // 32 vectors) until there are about 16 warps per SM; larger ones take whole rows
    const long long want = 16LL * sms;
    int nchunks = static_cast<int>((want + T - 1) / T);
    const int max_chunks = (vec + 31) / 32;
    if (nchunks > max_chunks) nchunks = max_chunks;
    if (nchunks < 1) nchunks = 1;
    const int chunk = ((vec + nchunks - 1) / nchunks + 31) / 32 * 32;
    const long long items = static_cast<long long>(T) * ((vec + chunk - 1) / chunk);
    long long blocks = (items + 7) / 8;
    const long long cap = static_cast<long long>(sms) * 8;
    if (blocks > cap) blocks = cap;
    return launch_k(gather_by_token_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s,
                    static_cast<const uint4*>(hidden), perm_dst, T, k, rows_max, vec,
                    chunk, static_cast<uint4*>(x_perm));
}

cudaError_t launch_gather(const void* hidden, const int32_t* perm_src, const int32_t* offsets,
                          int E, int T, int rows_max, int H, int elem_bytes, void* x_perm,
                          cudaStream_t s) {
    if (rows_max <= 0) return cudaSuccess;
    const int vec = H * elem_bytes / 16;
    int blocks = (rows_max + 7) / 8;
    const int cap = device_sm_count() * 8;
    if (blocks > cap) blocks = cap;
    return launch_k(gather_kernel, dim3(blocks), dim3(256), 0, s, static_cast<const uint4*>(hidden),
                    perm_src, offsets, E, T, rows_max, vec, static_cast<uint4*>(x_perm));
}

}  // namespace moe
