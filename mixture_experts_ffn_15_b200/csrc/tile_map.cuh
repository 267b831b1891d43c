// Tile map of a grouped GEMM: the groups (experts) own contiguous row ranges
// [offsets[g], offsets[g+1]) of the permuted rows, and every group is cut into tiles
// of `unit_rows` rows.  Built in shared memory by one warp of every CTA straight from
// the device offsets, so the host never waits for the routing.
#pragma once

#include "common.cuh"

namespace moe {

// offsets: [G+1] device array, or nullptr for one group of `rows` rows.  Offsets
// outside [0, rows] or decreasing are clamped and reported in *err (kErrBadExpert).
// s_off: sanitised offsets (clamped to [0, rows], non-decreasing); s_pre[g]: first
// tile of group g; s_pre[G]: tile count.  Runs on one warp; lane l owns the kPer
// consecutive entries l*kPer ..; every loop has a compile-time trip count, so the
// per-lane arrays stay in registers.
__device__ __forceinline__ void build_group_tiles(const int32_t* offsets, int rows, int32_t* err,
                                                  int G, int unit_rows, int* s_off, int* s_pre,
                                                  int lane) {
    constexpr int kPer = (kMaxExperts + 1 + 31) / 32;   // 9
    int v[kPer];
    bool bad = false;
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
        const int i = lane * kPer + q;
        int raw = rows;
        if (i <= G) raw = offsets ? offsets[i] : (i == 0 ? 0 : rows);
        if (i == 0 && offsets && raw != 0) bad = true;
        int c = raw < 0 ? 0 : (raw > rows ? rows : raw);
        if (c != raw) bad = true;
        v[q] = c;
    }
#pragma unroll
    for (int q = 1; q < kPer; ++q)
        if (v[q] < v[q - 1]) {
            bad = bad || (lane * kPer + q <= G);
            v[q] = v[q - 1];
        }
    int inc = v[kPer - 1];
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, inc, d);
        if (lane >= d) inc = max(inc, y);
    }
    int excl = __shfl_up_sync(0xffffffffu, inc, 1);
    if (lane == 0) excl = 0;
    // tiles of group g = lane*kPer + q: from the clamped offsets g and g + 1 (the
    // latter is the next entry, or the first entry of the next lane)
    const int first_next = __shfl_down_sync(0xffffffffu, max(v[0], excl), 1);
    int cnt[kPer];
    int lsum = 0;
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
        const int i = lane * kPer + q;
        if (v[q] < excl && i <= G) bad = true;
        v[q] = max(v[q], excl);
        if (i <= G) s_off[i] = v[q];
    }
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
        const int g = lane * kPer + q;
        const int hi = (q + 1 < kPer) ? v[q + 1 < kPer ? q + 1 : q] : first_next;
        int c = 0;
        if (g < G) c = (hi - v[q] + unit_rows - 1) / unit_rows;
        cnt[q] = c;
        lsum += c;
    }
    int incl = lsum;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += y;
    }
    int run = incl - lsum;
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
        const int g = lane * kPer + q;
        if (g <= G) s_pre[g] = run;   // g == G: the tile count
        run += cnt[q];
    }
    if (bad && offsets && err) atomicOr(err, kErrBadExpert);
    __syncwarp();
}

// Group of tile `tile` by binary search over s_pre.
__device__ __forceinline__ int tile_group(int tile, int G, const int* s_pre) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_pre[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    return lo;
}

}  // namespace moe
