// Router on the tensor cores (sm_100a) with the routing in the epilogue.
//
// "Gemma 4 MoE: re-enable fused com.microsoft::MoE op - #326", "Attribute set": k =
// top_k, normalize_routing_weights.  logits[t, e] = hidden[t] . router_w[e] (+ bias),
// 128-token tiles on the MMA's M side and all E experts on N; the epilogue selects,
// weighs and counts (per-tile bincount of "Contributing Gemma 4 support and ONNX
// export optimizations", "Key Technical Contributions").  One CTA per tile
// (tc_gemm_kernel<TOK_ROUTE>, persistent over the tiles), or a cluster of CTAs per tile
// splitting K (tc_route_split_kernel) when the batch has few tiles.
//
// Every wait is bounded (2 s); on expiry the CTA winds down, reports
// MOE_DEVERR_TIMEOUT in the error word and still frees its TMEM.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tc_common.cuh"
#include "tmap.cuh"
#include "topk_warp.cuh"

namespace moe {
namespace {

using namespace sm100;
using namespace tc;

// Routing of one 128-token tile from its logits in TMEM (columns 0..E-1, thread =
// token row).  Each thread keeps the KS = k+1 (or more) largest biased logits in a
// register list sorted descending, inserting the experts in index order so that equal
// logits keep the lower index first; then the softmax weights over the chosen k (or,
// normalize = 0, over all E), the near-tie flags, and the tile's bincount: per warp in
// shared memory (s_cnt is this warp's [E] slice), then added to tile_counts.
template <int E, int KS>
__device__ __forceinline__ void route_epilogue(uint32_t tb, bool valid, size_t row, int tile,
                                               const RouteParams& rp, const float* s_bias,
                                               int* s_cnt, int lane) {
    const int k = rp.k;
    float vals[KS];
    int ids[KS];
#pragma unroll
    for (int j = 0; j < KS; ++j) {
        vals[j] = -INFINITY;
        ids[j] = -1;
    }
#pragma unroll 1
    for (int c = 0; c < E; c += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tb + c, v);
        tmem_wait_ld();
        float x[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = f32(v[i]) + s_bias[c + i];
        if (valid && rp.logits) {
            uint4* dst = reinterpret_cast<uint4*>(rp.logits + row * E + c);
#pragma unroll
            for (int q = 0; q < 8; ++q)
                dst[q] = make_uint4(__float_as_uint(x[4 * q]), __float_as_uint(x[4 * q + 1]),
                                    __float_as_uint(x[4 * q + 2]), __float_as_uint(x[4 * q + 3]));
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const float xv = x[i];
            if (xv > vals[KS - 1]) {
                const int e = c + i;
#pragma unroll
                for (int j = KS - 1; j >= 0; --j) {
                    if (vals[j] < xv) {
                        if (j == 0 || vals[j - 1] >= xv) {
                            vals[j] = xv;
                            ids[j] = e;
                        } else {
                            vals[j] = vals[j - 1];
                            ids[j] = ids[j - 1];
                        }
                    }
                }
            }
        }
    }
    // rows past the batch hold bias-only logits (their A rows were zero-filled): finite
    const float vmax = vals[0];
    float den = 0.f;
    if (rp.normalize) {
#pragma unroll
        for (int j = 0; j < KS; ++j)
            if (j < k) den += expf(vals[j] - vmax);
    } else {
        // softmax over all E: a second, warp-uniform pass over the logits in TMEM
#pragma unroll 1
        for (int c = 0; c < E; c += 32) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(tb + c, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) den += expf(f32(v[i]) + s_bias[c + i] - vmax);
        }
    }
    if (valid) {
        int flags = 0;
        float kth = 0.f, next = -INFINITY;
#pragma unroll
        for (int j = 0; j < KS; ++j) {
            if (j < k) {
                rp.topk_idx[row * k + j] = ids[j];
                rp.topk_w[row * k + j] = expf(vals[j] - vmax) / den;
                atomicAdd(&s_cnt[ids[j]], 1);
                if (j + 1 < k && vals[j] - vals[j + 1] < kNearTieGap) flags |= 2;
            }
            if (j == k - 1) kth = vals[j];
            if (j == k) next = vals[j];
        }
        if (k < E && kth - next < kNearTieGap) flags |= 1;
        if (rp.near_tie) rp.near_tie[row] = flags;
    }
    // this warp's 32 rows: add its counts to the tile's (zeroed before the launch) and
    // clear them for the next tile; warp-local, so a warp that gave up on a wait never
    // holds the others at a barrier
    __syncwarp();
    for (int e = lane; e < E; e += 32) {
        const int c = s_cnt[e];
        if (c) {
            if (rp.tile_counts) atomicAdd(&rp.tile_counts[static_cast<size_t>(tile) * E + e], c);
            s_cnt[e] = 0;
        }
    }
    __syncwarp();
}

// Both router kernels signal their ring in stages of kRSub consecutive 64-K slots: a
// wait on an mbarrier costs the MMA thread ~160 cycles even on a completed phase and a
// commit ~90, more than the four N = 64 MMAs of one slot take on the tensor cores.
constexpr int kRSub = 2;

template <int MODE, int BN, int KS = 1>
__global__ void __launch_bounds__(kThreads, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const TcParams p, const RouteParams rp) {
    using C = Tr<MODE, BN>;
    static_assert(!C::kWeightM, "weight rows on M run in tc_ffn_decode_kernel");
    constexpr int kBars = C::kStages / kRSub;   // barrier stages of the slot ring
    static_assert(kBars * kRSub == C::kStages && kBars >= 2, "whole stages");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + C::kStages * C::kABytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(sB + C::kStages * C::kBBytes);
    uint64_t* empty = full + C::kStages;
    uint64_t* tfull = empty + C::kStages;
    uint64_t* tempty = tfull + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* s_off = reinterpret_cast<int*>(tmem_slot + 4);
    int* s_pre = s_off + (kMaxExperts + 1);
    float* s_bias = reinterpret_cast<float*>(s_pre + (kMaxExperts + 1));   // TOK_ROUTE
    int* s_cnt = reinterpret_cast<int*>(s_bias + kMaxExperts);            // TOK_ROUTE

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.offsets ? p.E : 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kBars; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tfull[a]), 1);
            mbar_init(smem_u32(&tempty[a]), 4);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
        tmem_relinquish();
    }
    // the prologue above touches no global memory; everything below may
    pdl_wait();
    pdl_trigger();
    if (warp == 2) build_tile_map(p, G, BM, s_off, s_pre, lane);
    if constexpr (MODE == TOK_ROUTE) {
        for (int e = threadIdx.x; e < BN; e += kThreads) s_bias[e] = rp.bias ? rp.bias[e] : 0.f;
        for (int e = threadIdx.x; e < 4 * BN; e += kThreads) s_cnt[e] = 0;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int per_unit = p.n_out / BN;
    const int num_units = s_pre[G] * per_unit;
    const int nk = p.K / BK;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            for (int u = blockIdx.x; u < num_units && !*abort_flag; u += gridDim.x) {
                const Unit t = decode_unit(u, per_unit, G, BM, s_off, s_pre);
                const uint32_t bytes = C::kStageBytes;
                const int wrow = t.g * p.n_out + t.sub * BN;
                for (int k0 = 0; k0 < nk; k0 += kRSub) {
                    const int ns = min(kRSub, nk - k0);   // slots of this stage (the last may be short)
                    if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag, kWaitLimitNs)) break;
                    const uint32_t fb = smem_u32(&full[stage]);
                    mbar_arrive_expect_tx(fb, static_cast<uint32_t>(ns) * bytes);
                    for (int j = 0; j < ns; ++j) {
                        const int sl = stage * kRSub + j, kb = k0 + j;
                        tma_load_2d(smem_u32(sA + sl * C::kABytes), &tmA, fb, kb * BK, t.row0);
                        tma_load_2d(smem_u32(sB + sl * C::kBBytes), &tmB, fb, kb * BK, wrow);
                    }
                    ++issued;
                    if (++stage == kBars) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (*abort_flag) {
                // let the copies already in flight land before the CTA exits
                int dummy = 0;
                for (int s = 0; s < kBars; ++s) {
                    if (issued <= s) break;
                    const long long fills = (issued - 1 - s) / kBars + 1;
                    mbar_wait(smem_u32(&full[s]), static_cast<uint32_t>((fills - 1) & 1),
                              &dummy, kWaitLimitNs / 4);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            for (int u = blockIdx.x; u < num_units && !*abort_flag; u += gridDim.x) {
                const Unit t = decode_unit(u, per_unit, G, BM, s_off, s_pre);
                const uint32_t idesc = idesc_bf16_f32(BM, BN);
                if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1u, abort_flag, kWaitLimitNs)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::kAccStride);
                bool ok = true;
                for (int k0 = 0; k0 < nk; k0 += kRSub) {
                    const int ns = min(kRSub, nk - k0);
                    if (!mbar_wait(smem_u32(&full[stage]), phase, abort_flag, kWaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    for (int j = 0; j < ns; ++j) {
                        const int sl = stage * kRSub + j, kb = k0 + j;
                        const uint32_t a0 = smem_u32(sA + sl * C::kABytes);
                        const uint32_t b0 = smem_u32(sB + sl * C::kBBytes);
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
                            umma_bf16(d_tmem, smem_desc_sw128(a0 + kk * 32), smem_desc_sw128(b0 + kk * 32),
                                      idesc, (kb | kk) != 0);
                    }
                    umma_commit(smem_u32(&empty[stage]));
                    if (++stage == kBars) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(smem_u32(&tfull[acc]));
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int quad = warp & 3;
        const int r = quad * 32 + lane;   // TMEM lane = row of the accumulator
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int u = blockIdx.x; u < num_units && !*abort_flag; u += gridDim.x) {
            const Unit t = decode_unit(u, per_unit, G, BM, s_off, s_pre);
            if (!mbar_wait(smem_u32(&tfull[acc]), acc_phase, abort_flag, kWaitLimitNs)) break;
            tc_fence_after();
            const uint32_t tb =
                tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(acc * C::kAccStride);
            const bool valid = r < t.nrows;
            const size_t orow = static_cast<size_t>(t.row0 + r);
            route_epilogue<BN, KS>(tb, valid, orow, t.row0 / BM, rp, s_bias,
                                   s_cnt + quad * BN, lane);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&tempty[acc]));
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
    if (threadIdx.x == 0 && *abort_flag && p.err) atomicOr(p.err, kErrTimeout);
}

// Routing of one token row from its E raw logits in shared memory (one thread): the
// KS = k+1 (or more) largest biased logits in a register list sorted descending,
// experts inserted in index order so that equal logits keep the lower index first;
// softmax weights over the chosen k (normalize) or over all E, near-tie flags, and the
// row's k counts added to the tile's bincount.
template <int E, int KS>
__device__ __forceinline__ void route_row(const float* logit, const float* s_bias, size_t row,
                                          int tile, const RouteParams& rp) {
    const int k = rp.k;
    float vals[KS];
    int ids[KS];
#pragma unroll
    for (int j = 0; j < KS; ++j) {
        vals[j] = -INFINITY;
        ids[j] = -1;
    }
    // 32 logits at a time into registers first: the insertion chain then runs on
    // registers, not on a shared-memory load per step
    static_assert(E % 32 == 0, "logit chunks");
#pragma unroll 1
    for (int c = 0; c < E; c += 32) {
        float x[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = logit[c + i] + s_bias[c + i];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const float xv = x[i];
            if (xv > vals[KS - 1]) {
                const int e = c + i;
#pragma unroll
                for (int j = KS - 1; j >= 0; --j) {
                    if (vals[j] < xv) {
                        if (j == 0 || vals[j - 1] >= xv) {
                            vals[j] = xv;
                            ids[j] = e;
                        } else {
                            vals[j] = vals[j - 1];
                            ids[j] = ids[j - 1];
                        }
                    }
                }
            }
        }
    }
    const float vmax = vals[0];
    float den = 0.f;
    if (rp.normalize) {
#pragma unroll
        for (int j = 0; j < KS; ++j)
            if (j < k) den += expf(vals[j] - vmax);
    } else {
#pragma unroll 1
        for (int c = 0; c < E; c += 32) {
            float x[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) x[i] = logit[c + i] + s_bias[c + i];
#pragma unroll
            for (int i = 0; i < 32; ++i) den += expf(x[i] - vmax);
        }
    }
    int flags = 0;
    float kth = 0.f, next = -INFINITY;
#pragma unroll
    for (int j = 0; j < KS; ++j) {
        if (j < k) {
            rp.topk_idx[row * k + j] = ids[j];
            rp.topk_w[row * k + j] = expf(vals[j] - vmax) / den;
            if (rp.tile_counts) atomicAdd(&rp.tile_counts[static_cast<size_t>(tile) * E + ids[j]], 1);
            if (j + 1 < k && vals[j] - vals[j + 1] < kNearTieGap) flags |= 2;
        }
        if (j == k - 1) kth = vals[j];
        if (j == k) next = vals[j];
    }
    if (k < E && kth - next < kNearTieGap) flags |= 1;
    if (rp.near_tie) rp.near_tie[row] = flags;
}

// ------------------------------------------------------------------------ split-K router
// Router logits and routing for a few 128-token tiles (batched decode, mid-sized
// prefill), where one CTA per tile would stream the whole K range alone.  A cluster of
// CS CTAs runs one tile: CTA r accumulates the K slices [r nk / CS, (r + 1) nk / CS) on
// the tensor cores (128 tokens on M, all E experts on N).  CTA q reduces and routes rows
// q 128 / CS .. of the tile: every CTA stores each of its partial rows straight from
// tensor memory into the shared memory of the CTA that reduces it (16-byte stores
// through the cluster, one block per source rank), and one cluster barrier publishes
// them all.  CTA q then sums the CS partials of its rows in rank order 0 .. CS-1 (a
// fixed order: the logits do not depend on timing) into a [row][e] block and one thread
// per row routes it (a warp per row, with its k + 1 rounds of warp reductions, took
// 1.3 us a row).  After the barrier no CTA touches another's shared memory, so none
// waits for the others before leaving.  No global scratch; the host picks this kernel
// by (T, H, E) alone, for the staged router and the layer alike, so both return the
// same bits.
template <int E, int CS>
struct SplitCfg {
    static constexpr int kRows = BM / CS;                       // rows reduced and routed per CTA
    static constexpr int kABytes = BM * BK * 2;                 // 128 token rows x 64 K
    static constexpr int kBBytes = E * BK * 2;                  // E router rows x 64 K
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kRecvLd = E + 4;                       // floats a received row (padded)
    // received partials [CS source ranks][kRows rows][kRecvLd]: CS * kRows = BM rows
    static constexpr int kPartBytes = BM * kRecvLd * 4;
    static constexpr int kRedBytes = kRows * (E + 1) * 4 + E * 4;   // sums [row][e], padded; bias
    static constexpr int kStagesFit = (210 * 1024 - kPartBytes - kRedBytes) / kStageBytes;
    static constexpr int kStages = kStagesFit > 4 ? 4 : kStagesFit;
    // barriers (full, empty: kStages each; tfull), then the TMEM slot and the abort flag
    static constexpr int kMiscBytes = (2 * kStages + 1) * 8 + 16;
    static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kPartBytes + kRedBytes + kMiscBytes;
    static constexpr int kTmemCols = E;                         // 64 or 128
    static_assert(kStages >= 2, "pipeline");
    static_assert(kRows % 4 == 0, "16-byte row groups");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

template <int E, int CS, int KS>
__global__ void __launch_bounds__(kThreads, 1)
tc_route_split_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const TcParams p, const RouteParams rp) {
    using C = SplitCfg<E, CS>;
    // slots per barrier stage: two where the ring holds an even number of at least 4
    constexpr int kSub = (C::kStages % 2 == 0 && C::kStages >= 4) ? kRSub : 1;
    constexpr int kBars = C::kStages / kSub;
    static_assert(kBars * kSub == C::kStages && kBars >= 2, "whole stages");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + C::kStages * C::kABytes;
    float* recv = reinterpret_cast<float*>(sB + C::kStages * C::kBBytes);   // [CS][kRows][kRecvLd]
    float* red = recv + BM * C::kRecvLd;                                    // [kRows][E + 1]
    float* s_bias = red + C::kRows * (E + 1);                               // [E]
    uint64_t* full = reinterpret_cast<uint64_t*>(s_bias + E);
    uint64_t* empty = full + C::kStages;
    uint64_t* tfull = empty + C::kStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tfull + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rank = static_cast<int>(cluster_ctarank());
    const int tile = static_cast<int>(blockIdx.x) / CS;
    const int nk = p.K / BK;
    const int kb0 = nk * rank / CS, kb1 = nk * (rank + 1) / CS;   // CS <= nk: never empty

    if (threadIdx.x == 0) {
        for (int s = 0; s < kBars; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        mbar_init(smem_u32(tfull), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
        tmem_relinquish();
    }
    // the prologue above touches no global memory; everything below may
    pdl_wait();
    pdl_trigger();
    for (int e = threadIdx.x; e < E; e += kThreads) s_bias[e] = rp.bias ? rp.bias[e] : 0.f;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            for (int k0 = kb0; k0 < kb1; k0 += kSub) {
                const int ns = min(kSub, kb1 - k0);
                if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag, kWaitLimitNs)) break;
                const uint32_t fb = smem_u32(&full[stage]);
                mbar_arrive_expect_tx(fb, static_cast<uint32_t>(ns) * C::kStageBytes);
                for (int j = 0; j < ns; ++j) {
                    const int sl = stage * kSub + j, kb = k0 + j;
                    tma_load_2d(smem_u32(sA + sl * C::kABytes), &tmA, fb, kb * BK, tile * BM);
                    tma_load_2d(smem_u32(sB + sl * C::kBBytes), &tmB, fb, kb * BK, 0);
                }
                ++issued;
                if (++stage == kBars) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (*abort_flag) {
                // let the copies already in flight land before the CTA goes on
                int dummy = 0;
                for (int s2 = 0; s2 < kBars; ++s2) {
                    if (issued <= s2) break;
                    const long long fills = (issued - 1 - s2) / kBars + 1;
                    mbar_wait(smem_u32(&full[s2]), static_cast<uint32_t>((fills - 1) & 1), &dummy,
                              kWaitLimitNs / 4);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(BM, E);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int k0 = kb0; k0 < kb1; k0 += kSub) {
                const int ns = min(kSub, kb1 - k0);
                if (!mbar_wait(smem_u32(&full[stage]), phase, abort_flag, kWaitLimitNs)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int j = 0; j < ns; ++j) {
                    const int sl = stage * kSub + j, kb = k0 + j;
                    const uint32_t a0 = smem_u32(sA + sl * C::kABytes);
                    const uint32_t b0 = smem_u32(sB + sl * C::kBBytes);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        umma_bf16(tmem_base, smem_desc_sw128(a0 + kk * 32), smem_desc_sw128(b0 + kk * 32),
                                  idesc, (kb != kb0 || kk != 0) ? 1u : 0u);
                }
                umma_commit(smem_u32(&empty[stage]));
                if (++stage == kBars) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (ok) umma_commit(smem_u32(tfull));
        }
    } else {
        // ------------------------------------------------------------ partials
        // warps 2..5: TMEM lane quadrant warp % 4; thread = token row r of the tile.  The
        // row goes straight into the shared memory of the CTA that reduces it (rank
        // r / kRows), at recv[this rank][r % kRows]: 16-byte stores through the cluster.
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        const int owner = r / C::kRows, ri = r - owner * C::kRows;
        const uint32_t dst = mapa_shared(smem_u32(recv + (rank * C::kRows + ri) * C::kRecvLd),
                                         static_cast<uint32_t>(owner));
        if (mbar_wait(smem_u32(tfull), 0, abort_flag, kWaitLimitNs)) {
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < E; c += 32) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + c, v);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; i += 4)
                    st_shared_cluster_v4(dst + (c + i) * 4, __uint_as_float(v[i]), __uint_as_float(v[i + 1]),
                                         __uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]));
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    // every CTA's partials have landed where they are reduced: after this barrier no CTA
    // touches another's shared memory, so none waits for the others again before leaving
    cluster_sync();

    // ---------------------------------------------------------------- reduce and route
    // row i, experts 4 q .. 4 q + 3: the CS received partials summed in rank order 0 ..
    // CS-1 (a fixed order: the logits do not depend on timing)
    const int row0 = rank * C::kRows;
#pragma unroll 1
    for (int pos = threadIdx.x; pos < C::kRows * (E / 4); pos += kThreads) {
        const int i = pos / (E / 4), e = 4 * (pos - i * (E / 4));
        float4 sum = *reinterpret_cast<const float4*>(recv + i * C::kRecvLd + e);
#pragma unroll
        for (int q = 1; q < CS; ++q) {
            const float4 v = *reinterpret_cast<const float4*>(recv + (q * C::kRows + i) * C::kRecvLd + e);
            sum.x += v.x;
            sum.y += v.y;
            sum.z += v.z;
            sum.w += v.w;
        }
        red[i * (E + 1) + e + 0] = sum.x;
        red[i * (E + 1) + e + 1] = sum.y;
        red[i * (E + 1) + e + 2] = sum.z;
        red[i * (E + 1) + e + 3] = sum.w;
    }
    __syncthreads();
    if (rp.logits) {   // the staged router returns the logits it selected on
#pragma unroll 1
        for (int i = warp; i < C::kRows; i += kThreads / 32) {
            const size_t row = static_cast<size_t>(tile) * BM + row0 + i;
            if (row < static_cast<size_t>(p.rows))
                for (int e = lane; e < E; e += 32) rp.logits[row * E + e] = red[i * (E + 1) + e] + s_bias[e];
        }
    }
    // one thread per row: the k + 1 (or more) largest biased logits in a descending
    // register list, as in the one-CTA-per-tile router's epilogue
    if (threadIdx.x < C::kRows) {
        const int i = threadIdx.x;
        const size_t row = static_cast<size_t>(tile) * BM + row0 + i;
        if (row < static_cast<size_t>(p.rows)) route_row<E, KS>(red + i * (E + 1), s_bias, row, tile, rp);
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
    if (threadIdx.x == 0 && *abort_flag && p.err) atomicOr(p.err, kErrTimeout);
}


// ------------------------------------------------------------------------ host side


template <int MODE, int BN, int KS = 1>
cudaError_t launch_one(const CUtensorMap& a, const CUtensorMap& b, const TcParams& p, int bound,
                       cudaStream_t s, const RouteParams& rp = RouteParams{}) {
    using C = Tr<MODE, BN>;
    auto kern = tc_gemm_kernel<MODE, BN, KS>;
    // once per device (outside any stream capture: the first call of every path
    // runs eagerly before a graph is captured)
    static bool attr_set[64] = {false};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    int grid = device_sm_count();
    if (bound < grid) grid = bound;
    if (grid <= 0) return cudaSuccess;
    return launch_k(kern, dim3(grid), dim3(kThreads), C::kSmemBytes, s, a, b, p, rp);
}

// Cluster size of the split-K router for these sizes (1: the one-CTA-per-tile router).
// A pure function of the sizes (a fixed budget of 148 CTAs, not the device's count), so
// that the staged router and the layer take the same kernel and give the same bits.
int route_split_cluster(int T, int H, int E) {
    if (E != 64 && E != 128) return 1;
    const int tiles = (T + BM - 1) / BM, nk = H / BK;
    for (int cs = 8; cs >= 2; cs >>= 1)
        if (tiles * cs <= 148 && cs <= nk) return cs;
    return 1;
}

template <int E, int CS, int KS>
cudaError_t launch_route_split(const CUtensorMap& a, const CUtensorMap& b, const TcParams& p,
                               const RouteParams& rp, int tiles, cudaStream_t s) {
    using C = SplitCfg<E, CS>;
    auto kern = tc_route_split_kernel<E, CS, KS>;
    static bool attr_set[64] = {false};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(tiles * CS));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    count_launch();
    return cudaLaunchKernelEx(&cfg, kern, a, b, p, rp);
}

}  // namespace

bool tc_route_supported(int H, int E, int k) {
    return H % 64 == 0 && (E == 64 || E == 128 || E == 256) && k >= 1 && k <= 32;
}

cudaError_t launch_route_tc(const void* hidden, const void* router_w, const float* bias, int T,
                            int H, int E, int k, int normalize, int32_t* topk_idx, float* topk_w,
                            int32_t* near_tie, float* logits, int32_t* tile_counts, int32_t* err,
                            cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    TcParams p{nullptr, 1, T, H, E, nullptr, E, err};
    RouteParams rp{bias, k, normalize ? 1 : 0, topk_idx, topk_w, near_tie, logits, tile_counts};
    CUtensorMap ma, mb;
    if (!tmap::matrix(&ma, hidden, T, H, BM)) return cudaErrorInvalidValue;
    if (!tmap::matrix(&mb, router_w, E, H, E)) return cudaErrorInvalidValue;
    const int cs = route_split_cluster(T, H, E);
    const int tiles = (T + BM - 1) / BM;
    if (cs > 1) {
#define MOE_SPLIT_CASE(EV, CV)                                                            \
    if (E == EV && cs == CV)                                                              \
        return k <= 8 ? launch_route_split<EV, CV, 9>(ma, mb, p, rp, tiles, s)             \
                      : launch_route_split<EV, CV, 33>(ma, mb, p, rp, tiles, s);
        MOE_SPLIT_CASE(64, 2) MOE_SPLIT_CASE(64, 4) MOE_SPLIT_CASE(64, 8)
        MOE_SPLIT_CASE(128, 2) MOE_SPLIT_CASE(128, 4) MOE_SPLIT_CASE(128, 8)
#undef MOE_SPLIT_CASE
        return cudaErrorInvalidValue;
    }
    const int bound = (T + BM - 1) / BM;
    const bool small_k = k <= 8;
#define MOE_ROUTE_CASE(EV)                                                                   \
    case EV:                                                                                 \
        return small_k ? launch_one<TOK_ROUTE, EV, 9>(ma, mb, p, bound, s, rp)               \
                       : launch_one<TOK_ROUTE, EV, 33>(ma, mb, p, bound, s, rp);
    switch (E) {
        MOE_ROUTE_CASE(64)
        MOE_ROUTE_CASE(128)
        MOE_ROUTE_CASE(256)
        default:
            return cudaErrorInvalidValue;
    }
#undef MOE_ROUTE_CASE
}

}  // namespace moe
