// Definitions shared by the single-CTA tcgen05 kernels (the router in route_tc.cu,
// the decode FFN in gemm_tc.cu): tile sizes, the tile-configuration traits, the
// parameter blocks and the unit decoding of a grouped tile list.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "tile_map.cuh"
#include "tmap.cuh"

namespace moe {
namespace tc {

constexpr int BM = 128;              // rows of A per tile (MMA M)
constexpr int BK = 64;               // K per stage: one 128-byte row of bf16
static_assert(BK == tmap::kBoxK, "TMA box width");
constexpr int kThreads = 192;
constexpr int kTokChunk = 64;        // weight-M: tokens per unit
constexpr int kBoxTok = 16;          // weight-M: token rows per TMA box
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// TOK_ROUTE: router logits with the routing itself in the epilogue (top-k, softmax,
// near-tie flags, per-tile bincount).
enum Mode : int { W_PLAIN = 4, TOK_ROUTE = 5 };

template <int MODE, int BN>
struct Tr {
    static constexpr bool kWeightM = (MODE == W_PLAIN);
    static constexpr int kBRows = kWeightM ? kTokChunk : BN;
    static constexpr int kABytes = BM * BK * 2;
    static constexpr int kBBytes = kBRows * BK * 2;
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kStagesFit = (200 * 1024) / kStageBytes;
    static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
    static constexpr int kAccStride = kWeightM ? kTokChunk : 256;
    static constexpr int kTmemCols = kWeightM ? 128 : 512;
    // barriers, tmem slot + abort flag, offsets, prefix, gather rows of one chunk
    static constexpr int kMiscBytes =
        (2 * kStages + 4) * 8 + 16 + 2 * (kMaxExperts + 1) * 4 + 16 * 8 + 64 +
        (MODE == TOK_ROUTE ? 5 * kMaxExperts * 4 : 0);   // bias [E], counts [4][E]
    static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kMiscBytes;
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
    static_assert(kWeightM || (BN % 16 == 0 && BN >= 16 && BN <= 256), "UMMA N");
};

struct TcParams {
    const int32_t* offsets;   // [E+1] device, or nullptr: one group of `rows` rows
    int E;
    int rows;                 // rows of the token matrix
    int K;                    // reduction length (multiple of 64)
    int n_out;                // weight rows per expert
    void* out;
    int ldo;                  // output row stride, elements
    int32_t* err;
};

// The routing half of TOK_ROUTE (n_out = number of experts).
struct RouteParams {
    const float* bias;        // [E] or nullptr
    int k, normalize;
    int32_t* topk_idx;        // [T, k]
    float* topk_w;            // [T, k]
    int32_t* near_tie;        // [T] or nullptr
    float* logits;            // [T, E] or nullptr (logits + bias)
    int32_t* tile_counts;     // [ceil(T / 128), E]
};

struct Unit {
    int g;      // expert
    int row0;   // first token row
    int nrows;  // valid token rows (<= kUnitRows)
    int sub;    // column tile (token-M) or weight row tile (weight-M) inside the expert
};

__device__ __forceinline__ void build_tile_map(const TcParams& p, int G, int unit_rows, int* s_off,
                                               int* s_pre, int lane) {
    build_group_tiles(p.offsets, p.rows, p.err, G, unit_rows, s_off, s_pre, lane);
}

__device__ __forceinline__ Unit decode_unit(int u, int per_unit, int G, int unit_rows,
                                            const int* s_off, const int* s_pre) {
    const int tile = u / per_unit;
    Unit t;
    t.sub = u - tile * per_unit;
    int lo = 0, hi = G - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_pre[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    t.g = lo;
    t.row0 = s_off[lo] + (tile - s_pre[lo]) * unit_rows;
    t.nrows = min(unit_rows, s_off[lo + 1] - t.row0);
    return t;
}

__device__ __forceinline__ float f32(uint32_t x) { return __uint_as_float(x); }

}  // namespace tc
}  // namespace moe
