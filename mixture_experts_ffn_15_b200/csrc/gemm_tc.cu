// Decode FFN on the tensor cores (sm_100a): the grouped matmul of grouped_mm_experts_forward for batches with few
// rows per expert, fc1 + SwiGLU and fc2 (standard SwiGLU, interleaved fc1) in one
// persistent launch with 128 weight rows on M and the expert's tokens on N, so that
// every weight byte streams from HBM once; optionally with the routing and the
// weighted combine inside the same launch.
//
// One persistent CTA per SM, 6 warps:
//   warp 0     TMA producer: A and B tiles (64-wide K slices, 128-byte swizzle)
//              into a ring of shared-memory stages, completion on mbarriers;
//   warp 1     MMA issuer: tcgen05.mma kind::f16 (bf16 x bf16 -> f32) into one of
//              two TMEM accumulators, tcgen05.commit frees stages / publishes tiles;
//   warps 2-5  epilogue: tcgen05.ld of the accumulator (warp w reads TMEM lanes
//              32*(w%4) .. +31).  The second accumulator lets the epilogue of one
//              tile overlap the next mainloop.
// Tile maps are rebuilt in every CTA from device offsets (no host sync).
//
// Every wait is bounded (2 s); on expiry the CTA winds down, reports
// MOE_DEVERR_TIMEOUT in the error word and still frees its TMEM.
#include <cuda.h>

#include <atomic>

#include "combine.cuh"
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tc_common.cuh"
#include "tile_map.cuh"
#include "tmap.cuh"
#include "topk_warp.cuh"

namespace moe {
namespace {

using namespace sm100;
using namespace tc;

// ------------------------------------------------------------------------ decode FFN
// fc1 + SwiGLU and fc2 for batches with few rows per expert, in ONE persistent
// launch.  Both GEMMs put 128 weight rows on the MMA's M side and the expert's tokens
// (a chunk of at most 64 permuted rows) on N, so every weight byte streams from HBM
// once.  The unit list holds every fc1 unit (chunk x 128 rows of fc1) and then every
// fc2 unit (chunk x 128 rows of fc2).  A CTA's first unit is unit blockIdx.x; later
// ones come in list order from a global counter starting at gridDim.x (the producer
// warp claims -- with int8 experts the int8 producer, which runs furthest ahead -- and
// a 4-slot ring in shared memory hands the unit to the other warps), so the large fc1
// units go first and the small fc2 units even out the end, and no CTA waits on the
// counter's atomic before its first load.  An fc2 unit is handed out only after every
// fc1 unit is some running CTA's (first units are taken before any wait).  An fc2 unit needs the
// activations of its chunk: each fc1 epilogue warp publishes its stores with a proxy
// fence and a release increment of the chunk's counter, and the fc2 producer waits
// (bounded) for 4 x (fc1 units per chunk) increments with an acquire load before
// loading the activations with TMA.  The fc2 weights of a unit do not depend on fc1.
// With GATHER, fc1's token rows come straight from `hidden` through perm_src (four rows
// per tile::gather4 load); otherwise from contiguous rows of x_perm (16-row boxes).
// With `out`, the kernel also does the weighted combine: once every fc2 unit has
// published its rows (a grid-wide count, acquire), the epilogue warps of all CTAs
// split the output vectors among themselves, with the same arithmetic as
// combine_kernel.
// Every CTA of the grid (at most one per SM) is resident, so the waits always end.
constexpr int kUnitRing = 4;

// Weight-only int8 experts (Q8): the weights stream from HBM as int8 through a deep ring
// of their own (kQStages tiles of 128 rows x 64 bytes, loaded by a dedicated producer
// warp); converter warps turn each tile into bf16 -- exact, |q| <= 127 -- and store it
// straight into tensor memory, where the MMA reads its A operand (two groups of four
// warps taking alternate stages, so that two stages convert at once); shared memory
// carries only int8 weights and token rows.  The epilogue multiplies each weight row's
// accumulator by its float32 scale.  The token side is the bf16 path's.
constexpr int kQBytes = BM * BK;   // one int8 tile: 128 weight rows x 64 K

template <bool Q8>
struct DecodeCfg {
    using T = Tr<W_PLAIN, 64>;
    static constexpr int kABytes = Q8 ? 0 : T::kABytes;     // Q8: A lives in tensor memory
    static constexpr int kBBytes = T::kBBytes;
    // The ring holds kSlots 64-K slots (A in shared or tensor memory + token B); the
    // barriers work on stages of kSub consecutive slots, so that every wait and commit
    // of the MMA thread covers 4 kSub MMAs: a wait on an mbarrier costs the issuing
    // thread ~160 cycles even when the phase has completed, and a commit ~90, against
    // ~60 for an M = 128, N <= 64, K = 16 MMA.
    static constexpr int kSlots = T::kStages;
    static constexpr int kSub = 2;
    static constexpr int kStages = kSlots / kSub;
    static_assert(kStages * kSub == kSlots, "whole stages");
    static constexpr int kQStages = Q8 ? 16 : 0;            // int8 weight ring
    static constexpr int kThreads = Q8 ? 480 : 192;         // + Q producer + 2 x 4 converters
    static constexpr int kAccStride = T::kAccStride;
    // Q8: two accumulators (2 x 64 columns), then one A stage of 32 columns per ring stage
    static constexpr int kTmemA = 2 * kAccStride;
    static constexpr int kTmemCols = Q8 ? 512 : T::kTmemCols;
    static_assert(!Q8 || kTmemA + kSlots * 32 <= kTmemCols, "tensor memory");
    static constexpr int kDataBytes = kSlots * (kABytes + kBBytes) + kQStages * kQBytes;
    static constexpr int kMiscBytes = T::kMiscBytes + 2 * kQStages * 8;   // + int8 ring barriers
    static constexpr int kSmemBytes = 1024 + kDataBytes + kMiscBytes;
    static_assert(kStages <= T::kStages, "barrier space");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

struct DecodeParams {
    const int32_t* offsets;   // [E+1]
    const int32_t* perm_src;  // [rows] with GATHER, else nullptr
    int E, rows, T, H, I;
    __nv_bfloat16* act;       // [rows, I]
    __nv_bfloat16* y;         // [rows, H]
    int32_t* done;            // one counter per chunk, zero on entry
    int32_t* sched;           // units claimed past the first gridDim.x, zero on entry
    int32_t* fc2_done;        // published fc2 units (x 4 warps), zero on entry
    // fused combine (out != nullptr): out[t] = sum_j topk_w[t, j] y[perm_dst[t*k + j]]
    const int32_t* perm_dst;
    const float* topk_w;
    int k;
    __nv_bfloat16* out;
    int32_t* err;
    SwigluAttr act_attr;            // SwiGLU attributes
    const __nv_bfloat16* b1;        // [E, 2I] fc1 bias (fc1's layout) or nullptr
    bool fc1_chunked;               // fc1 and b1 in the chunked layout
    const __nv_bfloat16* b2;        // [E, H] fc2 bias or nullptr
    const float* s1;                // Q8: [E, 2I] fc1 row scales (fc1's layout)
    const float* s2;                // Q8: [E, H] fc2 row scales
    // ROUTE: the routing runs inside the launch (fields below); offsets, perm_src,
    // perm_dst and topk_w above are then unused (the kernel keeps them in shared memory)
    const void* hidden;       // [T, H]
    const void* router_w;     // [E, H]
    const float* bias;        // [E] or nullptr
    int normalize;
    float* logits;            // [T, E] scratch
    int32_t* route_bar;       // grid-barrier arrivals, zero on entry
    int route_bar_extra;      // arrivals wanted beyond the grid (0; 1 only to test a timeout)
    uint64_t route_wait_ns;   // limit of the grid-barrier wait
    // the routing as the staged calls would return it, written by CTA 0
    int32_t* r_topk_idx;      // [T, k]
    float* r_topk_w;          // [T, k]
    int32_t* r_near_tie;      // [T] or nullptr
    int32_t* r_counts;        // [E]
    int32_t* r_offsets;       // [E + 1]
    int32_t* r_perm_src;      // [T k]
    int32_t* r_perm_dst;      // [T k]
};

// Shared memory the in-kernel routing keeps for the whole launch (after the misc block).
constexpr int kRouteSmemBytes =
    4 * kFusedRouteMaxRows * 4 +                  // ids, weights, perm_dst, perm_src
    kMaxExperts * 4 + (kMaxExperts + 4) * 4 +     // counts, offsets
    kMaxExperts * (kFusedRouteMaxT / 32) * 4 +    // token masks per expert
    16 * 8 * 4;                                   // partial dot products (<= 16 warps)

__device__ __forceinline__ int ld_acquire(const int32_t* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Two int8 weights held as float32 bit patterns 0x4B000000 | (b ^ 0x80) = 2^23 + 128 + b:
// subtract 2^23 + 128 from both with one packed add.rn.f32x2 (exact, the differences are
// the integers b) and pack the two upper halves -- b in bf16, exact for |b| <= 128 -- into
// one bf16x2 word, the first weight in the lower half.
__device__ __forceinline__ uint32_t sub_magic_f32x2(uint32_t a, uint32_t b) {
    uint64_t d;
    asm("{\n\t.reg .b64 x;\n\t"
        "mov.b64 x, {%1, %2};\n\t"
        "add.rn.f32x2 %0, x, %3;\n\t}"
        : "=l"(d)
        : "r"(a), "r"(b), "l"(0xCB000080CB000080ull));   // -(2^23 + 128) in both halves
    return __byte_perm(static_cast<uint32_t>(d), static_cast<uint32_t>(d >> 32), 0x7632u);
}

__device__ __forceinline__ bool wait_count(const int32_t* ctr, int target, volatile int* abort,
                                           uint64_t limit_ns = kWaitLimitNs) {
    if (ld_acquire(ctr) >= target) return true;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
        __nanosleep(64);
        if (ld_acquire(ctr) >= target) return true;
        if (*abort) return false;
        if (global_timer_ns() - t0 > limit_ns) {
            *abort = 1;
            return false;
        }
    }
}

struct DUnit {
    int phase;   // 1: fc1 + SwiGLU, 2: fc2
    int chunk;
    int g, row0, nrows, mt;
};

__device__ __forceinline__ DUnit decode_dunit(int u, int U1, int MT1, int MT2, int G,
                                              const int* s_off, const int* s_pre) {
    DUnit d;
    int v, MT;
    if (u < U1) {
        d.phase = 1;
        v = u;
        MT = MT1;
    } else {
        d.phase = 2;
        v = u - U1;
        MT = MT2;
    }
    d.chunk = v / MT;
    d.mt = v - d.chunk * MT;
    int lo = 0, hi = G - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_pre[mid] <= d.chunk) lo = mid; else hi = mid - 1;
    }
    d.g = lo;
    d.row0 = s_off[lo] + (d.chunk - s_pre[lo]) * kTokChunk;
    d.nrows = min(kTokChunk, s_off[lo + 1] - d.row0);
    return d;
}

template <bool GATHER, bool ROUTE, bool Q8>
__global__ void __launch_bounds__(DecodeCfg<Q8>::kThreads, 1)
tc_ffn_decode_kernel(const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ CUtensorMap tmX,
                     const __grid_constant__ CUtensorMap tmW2, const __grid_constant__ CUtensorMap tmAct,
                     const DecodeParams p) {
    using C = DecodeCfg<Q8>;
    static_assert(C::kThreads <= 16 * 32, "partial dot products of the routing");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + C::kSlots * C::kABytes;
    uint8_t* sQ = sB + C::kSlots * C::kBBytes;                // Q8: int8 weight ring
    uint64_t* full = reinterpret_cast<uint64_t*>(sQ + C::kQStages * kQBytes);
    uint64_t* empty = full + C::kStages;
    uint64_t* tfull = empty + C::kStages;
    uint64_t* tempty = tfull + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* s_off = reinterpret_cast<int*>(tmem_slot + 4);
    int* s_pre = s_off + (kMaxExperts + 1);
    int* s_unit = s_pre + (kMaxExperts + 1);                        // [kUnitRing]
    uint64_t* ufull = reinterpret_cast<uint64_t*>(s_unit + 2 * kUnitRing);   // 8-byte aligned
    uint64_t* uempty = ufull + kUnitRing;
    uint64_t* qfull = uempty + kUnitRing;                    // Q8: [kQStages]
    uint64_t* qempty = qfull + C::kQStages;
    // ROUTE only: the routing of the whole batch, after the misc block
    int* s_ridx = reinterpret_cast<int*>(smem + C::kDataBytes + C::kMiscBytes);
    float* s_rw = reinterpret_cast<float*>(s_ridx + kFusedRouteMaxRows);
    int* s_pdst = reinterpret_cast<int*>(s_rw + kFusedRouteMaxRows);
    int* s_psrc = s_pdst + kFusedRouteMaxRows;
    int* s_rcnt = s_psrc + kFusedRouteMaxRows;
    int* s_roff = s_rcnt + kMaxExperts;
    uint32_t* s_rmask = reinterpret_cast<uint32_t*>(s_roff + kMaxExperts + 4);
    float* s_red = reinterpret_cast<float*>(s_rmask + kMaxExperts * (kFusedRouteMaxT / 32));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.E;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            // Q8: the token producer's arrival (with its bytes) and the 4 converter warps
            mbar_init(smem_u32(&full[s]), Q8 ? 5 : 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tfull[a]), 1);
            mbar_init(smem_u32(&tempty[a]), 4);
        }
        for (int q = 0; q < kUnitRing; ++q) {
            mbar_init(smem_u32(&ufull[q]), 1);
            // the MMA thread and 4 epilogue warps (Q8: + the token producer and 8 converters;
            // the int8 producer claims)
            mbar_init(smem_u32(&uempty[q]), Q8 ? 14 : 5);
        }
        for (int q = 0; q < C::kQStages; ++q) {
            mbar_init(smem_u32(&qfull[q]), 1);
            mbar_init(smem_u32(&qempty[q]), 4);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmW1);
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmW2);
        tma_prefetch_desc(&tmAct);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
        tmem_relinquish();
    }
    // the prologue above touches no global memory; everything below may
    pdl_wait();
    pdl_trigger();
    if constexpr (ROUTE) {
        // ---------------------------------------------------------------- routing
        // (1) router logits: CTA c takes experts c, c + grid, ...; its 192 threads
        //     split H in 16-byte vectors (up to kR1Vec per thread and pass, all loads
        //     issued before the first product, so a pass costs one memory latency),
        //     8 tokens at a time; the partial sums are added warp by warp in a fixed
        //     order.
        constexpr int kR1Vec = 3;
        const int T = p.T, E = p.E, k = p.k;
        const int nv = p.H / 8;
        const uint4* x4 = reinterpret_cast<const uint4*>(p.hidden);
        const uint4 zero4 = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll 1
        for (int e = blockIdx.x; e < E; e += gridDim.x) {
            const uint4* w4 = reinterpret_cast<const uint4*>(p.router_w) + static_cast<size_t>(e) * nv;
#pragma unroll 1
            for (int t0 = 0; t0 < T; t0 += 8) {
                float acc[8];
#pragma unroll
                for (int t = 0; t < 8; ++t) acc[t] = 0.f;
#pragma unroll 1
                for (int v0 = threadIdx.x; v0 < nv; v0 += kR1Vec * C::kThreads) {
                    uint4 wv[kR1Vec], xv[8][kR1Vec];
#pragma unroll
                    for (int j = 0; j < kR1Vec; ++j) {
                        const int v = v0 + j * C::kThreads;
                        wv[j] = v < nv ? __ldg(w4 + v) : zero4;
#pragma unroll
                        for (int t = 0; t < 8; ++t)
                            xv[t][j] = (v < nv && t0 + t < T)
                                           ? __ldg(x4 + static_cast<size_t>(t0 + t) * nv + v)
                                           : zero4;
                    }
#pragma unroll
                    for (int j = 0; j < kR1Vec; ++j) {
                        float wf[8];
                        unpack_bf16x8(wv[j], wf);
#pragma unroll
                        for (int t = 0; t < 8; ++t) {
                            float xf[8];
                            unpack_bf16x8(xv[t][j], xf);
#pragma unroll
                            for (int i = 0; i < 8; ++i) acc[t] = fmaf(xf[i], wf[i], acc[t]);
                        }
                    }
                }
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    const float sum = warp_sum(acc[t]);
                    if (lane == 0) s_red[warp * 8 + t] = sum;
                }
                __syncthreads();
                if (threadIdx.x < 8 && t0 + static_cast<int>(threadIdx.x) < T) {
                    float sum = 0.f;
#pragma unroll
                    for (int w = 0; w < C::kThreads / 32; ++w) sum += s_red[w * 8 + threadIdx.x];
                    p.logits[static_cast<size_t>(t0 + threadIdx.x) * E + e] = sum;
                }
                __syncthreads();
            }
        }
        // (2) grid-wide barrier: the launch is cooperative (every CTA resident, at most
        //     one per SM), so the wait ends; it is bounded all the same (abort on expiry,
        //     before any bulk copy or MMA of this CTA is in flight).
        __syncthreads();
        if (threadIdx.x == 0) {
            __threadfence();
            atomicAdd(p.route_bar, 1);
            wait_count(p.route_bar, static_cast<int>(gridDim.x) + p.route_bar_extra, abort_flag,
                       p.route_wait_ns);
        }
        __syncthreads();
        // (3) every CTA selects, counts and places the whole batch itself (the same
        //     arithmetic everywhere, so every CTA holds the same routing); the logits
        //     are staged in the idle stage ring.
        float* s_log = reinterpret_cast<float*>(sA);
        {
            // all loads first, then the shared-memory stores (one L2 latency)
            constexpr int kR3Per = 8;
            for (int i0 = threadIdx.x; i0 < T * E; i0 += kR3Per * C::kThreads) {
                float lv[kR3Per];
#pragma unroll
                for (int j = 0; j < kR3Per; ++j) {
                    const int i = i0 + j * C::kThreads;
                    lv[j] = i < T * E ? __ldcg(p.logits + i) : 0.f;
                }
#pragma unroll
                for (int j = 0; j < kR3Per; ++j) {
                    const int i = i0 + j * C::kThreads;
                    if (i < T * E) s_log[i] = lv[j];
                }
            }
        }
        const int words = (T + 31) / 32;
        for (int i = threadIdx.x; i < E * words; i += C::kThreads) s_rmask[i] = 0;
        for (int e = threadIdx.x; e < E; e += C::kThreads) s_rcnt[e] = 0;
        __syncthreads();
        const bool lead = blockIdx.x == 0;
#pragma unroll 1
        for (int t = warp; t < T; t += C::kThreads / 32) {
            const WarpTopk r = warp_topk(s_log + t * E, p.bias, E, k, p.normalize, lane);
            if (lane < k) {
                s_ridx[t * k + lane] = r.idx;
                s_rw[t * k + lane] = r.w;
                if (static_cast<unsigned>(r.idx) < static_cast<unsigned>(E)) {
                    atomicAdd(&s_rcnt[r.idx], 1);
                    atomicOr(&s_rmask[r.idx * words + (t >> 5)], 1u << (t & 31));
                }
                if (lead) {
                    p.r_topk_idx[t * k + lane] = r.idx;
                    p.r_topk_w[t * k + lane] = r.w;
                }
            }
            if (lead && lane == 0 && p.r_near_tie) p.r_near_tie[t] = r.flags;
        }
        __syncthreads();
        if (warp == 0) {
            constexpr int per = kMaxExperts / 32;   // compile-time: loc[] stays in registers
            int loc[per];
            int lsum = 0;
#pragma unroll
            for (int q = 0; q < per; ++q) {
                const int e = lane * per + q;
                loc[q] = e < E ? s_rcnt[e] : 0;
                lsum += loc[q];
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
                    s_roff[e] = run;
                    if (lead) {
                        p.r_offsets[e] = run;
                        p.r_counts[e] = loc[q];
                    }
                }
                run += loc[q];
            }
            if (lane == 31) {
                s_roff[E] = incl;
                if (lead) p.r_offsets[E] = incl;
            }
        }
        __syncthreads();
        // stable placement: the rank of t among the tokens of its expert
        for (int q = threadIdx.x; q < T * k; q += C::kThreads) {
            const int e = s_ridx[q], t = q / k;
            int row = -1;
            if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) {
                const uint32_t* m = s_rmask + e * words;
                const int w = t >> 5;
                int rank = __popc(m[w] & ((1u << (t & 31)) - 1u));
                for (int i = 0; i < w; ++i) rank += __popc(m[i]);
                row = s_roff[e] + rank;
                s_psrc[row] = t;
                if (lead) p.r_perm_src[row] = t;
            }
            s_pdst[q] = row;
            if (lead) p.r_perm_dst[q] = row;
        }
        // the stage ring is written by TMA from here on
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncthreads();
    }
    if (warp == 2) {
        TcParams tp{ROUTE ? s_roff : p.offsets, p.E, p.rows, 0, 0, nullptr, 0, p.err};
        build_tile_map(tp, G, kTokChunk, s_off, s_pre, lane);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int MT1 = 2 * p.I / BM, MT2 = p.H / BM;
    const int CH = s_pre[G];
    const int U1 = CH * MT1;
    const int U = U1 + CH * MT2;
    const int nk1 = p.H / BK, nk2 = p.I / BK;
    const int fc1_done = 4 * MT1;   // increments per chunk: 4 epilogue warps per fc1 unit

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        // Lane 0 owns the barriers; every lane issues its share of the token rows.
        int stage = 0;
        uint32_t phase = 0;
        long long issued = 0;
        int slot = 0;
        uint32_t uphase = 0;
        int claims = 0;   // bf16: units this producer has claimed
        for (;;) {
            int u = U;
            if (lane == 0) {
                if constexpr (Q8) {
                    // the int8 producer claims; this warp reads the ring like the others
                    if (mbar_wait(smem_u32(&ufull[slot]), uphase, abort_flag, kWaitLimitNs)) {
                        u = s_unit[slot];
                        mbar_arrive(smem_u32(&uempty[slot]));
                    }
                } else {
                    if (mbar_wait(smem_u32(&uempty[slot]), uphase ^ 1u, abort_flag, kWaitLimitNs))
                        u = *abort_flag ? U
                            : claims++ == 0 ? static_cast<int>(blockIdx.x)
                                            : static_cast<int>(gridDim.x) + atomicAdd(p.sched, 1);
                    s_unit[slot] = u;
                    mbar_arrive(smem_u32(&ufull[slot]));
                }
            }
            u = __shfl_sync(0xffffffffu, u, 0);
            if (++slot == kUnitRing) {
                slot = 0;
                uphase ^= 1u;
            }
            if (u >= U) break;
            const DUnit d = decode_dunit(u, U1, MT1, MT2, G, s_off, s_pre);
            const bool f1 = d.phase == 1;
            const int nk = f1 ? nk1 : nk2;
            // both weight maps are (k, s, i, e) pair views: rows d.mt BM .. of expert d.g
            // (Q8: the int8 producer warp loads them)
            const CUtensorMap* ma = f1 ? &tmW1 : &tmW2;
            const int nl = (d.nrows + kBoxTok - 1) / kBoxTok;
            uint32_t bbytes = static_cast<uint32_t>(nl * kBoxTok * BK * 2);
            // gathered token rows: lane < nl4 loads rows 4 lane .. 4 lane + 3 of the chunk
            // (one tile::gather4 load; rows past the chunk repeat its last row)
            const int nl4 = (d.nrows + 3) / 4;
            int src[4] = {0, 0, 0, 0};
            if (f1 && GATHER) {
                if (lane < nl4) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int r = d.row0 + min(4 * lane + i, d.nrows - 1);
                        int t = ROUTE ? s_psrc[r] : p.perm_src[r];
                        if (t < 0 || t >= p.T) {
                            atomicOr(p.err, kErrBadExpert);
                            t = 0;
                        }
                        src[i] = t;
                    }
                }
                bbytes = static_cast<uint32_t>(nl4 * 4 * BK * 2);
            }
            if (!f1) {
                bool ok = true;
                if (lane == 0) ok = wait_count(&p.done[d.chunk], fc1_done, abort_flag);
                if (!__shfl_sync(0xffffffffu, ok, 0)) break;
                fence_proxy_async_global();
            }
            bool ok = true;
            for (int kb0 = 0; kb0 < nk; kb0 += C::kSub) {
                const int ns = min(C::kSub, nk - kb0);   // slots of this stage (the last may be short)
                if (lane == 0) {
                    ok = mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag, kWaitLimitNs);
                    if (ok)
                        mbar_arrive_expect_tx(smem_u32(&full[stage]),
                                              static_cast<uint32_t>(ns) * ((Q8 ? 0 : C::kABytes) + bbytes));
                }
                // the whole warp leaves together (lane 0 alone saw the wait give up)
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                const uint32_t fb = smem_u32(&full[stage]);
                for (int j = 0; j < ns; ++j) {
                    const int kb = kb0 + j, sl = stage * C::kSub + j;
                    const uint32_t a_dst = smem_u32(sA + sl * C::kABytes);
                    const uint32_t b_dst = smem_u32(sB + sl * C::kBBytes);
                    if (!Q8 && lane == 0) tma_load_4d(a_dst, ma, fb, kb * BK, 0, d.mt * (BM / 2), d.g);
                    if (f1 && GATHER) {
                        if (lane < nl4)
                            tma_gather4(b_dst + lane * 4 * BK * 2, &tmX, fb, kb * BK, src[0], src[1],
                                        src[2], src[3]);
                    } else if (lane < nl) {
                        tma_load_2d(b_dst + lane * kBoxTok * BK * 2, f1 ? &tmX : &tmAct, fb, kb * BK,
                                    d.row0 + lane * kBoxTok);
                    }
                }
                ++issued;
                if (++stage == C::kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
        }
        if (lane == 0 && *abort_flag) {
            // let the copies already in flight land before the CTA exits
            int dummy = 0;
            for (int s2 = 0; s2 < C::kStages; ++s2) {
                if (issued <= s2) break;
                const long long fills = (issued - 1 - s2) / C::kStages + 1;
                mbar_wait(smem_u32(&full[s2]), static_cast<uint32_t>((fills - 1) & 1), &dummy,
                          kWaitLimitNs / 4);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            int slot = 0;
            uint32_t uphase = 0;
            for (;;) {
                if (!mbar_wait(smem_u32(&ufull[slot]), uphase, abort_flag, kWaitLimitNs)) break;
                const int u = s_unit[slot];
                mbar_arrive(smem_u32(&uempty[slot]));
                if (++slot == kUnitRing) {
                    slot = 0;
                    uphase ^= 1u;
                }
                if (u >= U) break;
                const DUnit d = decode_dunit(u, U1, MT1, MT2, G, s_off, s_pre);
                const int nk = d.phase == 1 ? nk1 : nk2;
                const uint32_t idesc = idesc_bf16_f32(BM, ((d.nrows + 15) / 16) * 16);
                if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1u, abort_flag, kWaitLimitNs)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::kAccStride);
                bool ok = true;
                for (int kb0 = 0; kb0 < nk; kb0 += C::kSub) {
                    const int ns = min(C::kSub, nk - kb0);
                    if (!mbar_wait(smem_u32(&full[stage]), phase, abort_flag, kWaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    for (int j = 0; j < ns; ++j) {
                        const int kb = kb0 + j, sl = stage * C::kSub + j;
                        const uint32_t a0 = smem_u32(sA + sl * C::kABytes);
                        const uint32_t b0 = smem_u32(sB + sl * C::kBBytes);
                        if constexpr (Q8) {
                            // A: the converted slot in tensor memory, 8 columns per 16 K
                            const uint32_t at = tmem_base + static_cast<uint32_t>(C::kTmemA + sl * 32);
#pragma unroll
                            for (int kk = 0; kk < BK / 16; ++kk)
                                umma_bf16_ta(d_tmem, at + kk * 8, smem_desc_sw128(b0 + kk * 32), idesc,
                                             (kb | kk) != 0);
                        } else {
#pragma unroll
                            for (int kk = 0; kk < BK / 16; ++kk)
                                umma_bf16(d_tmem, smem_desc_sw128(a0 + kk * 32),
                                          smem_desc_sw128(b0 + kk * 32), idesc, (kb | kk) != 0);
                        }
                    }
                    umma_commit(smem_u32(&empty[stage]));
                    if (++stage == C::kStages) {
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
    } else if (warp < 6) {
        // ------------------------------------------------------------ epilogue
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        int slot = 0;
        uint32_t uphase = 0;
        for (;;) {
            const bool got = mbar_wait(smem_u32(&ufull[slot]), uphase, abort_flag, kWaitLimitNs);
            const int u = got ? s_unit[slot] : U;
            __syncwarp();
            if (got && lane == 0) mbar_arrive(smem_u32(&uempty[slot]));
            if (++slot == kUnitRing) {
                slot = 0;
                uphase ^= 1u;
            }
            if (u >= U) break;
            const DUnit d = decode_dunit(u, U1, MT1, MT2, G, s_off, s_pre);
            const bool f1 = d.phase == 1;
            if (!mbar_wait(smem_u32(&tfull[acc]), acc_phase, abort_flag, kWaitLimitNs)) break;
            tc_fence_after();
            const uint32_t tb = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                                static_cast<uint32_t>(acc * C::kAccStride);
            const int wr = d.mt * BM + r;   // weight row inside the expert
            // this lane's weight row's bias (fc1: interleaved row wr in fc1's layout, fc2: h)
            const __nv_bfloat16* bsrc = f1 ? p.b1 : p.b2;
            const size_t wi = static_cast<size_t>(d.g) * (f1 ? 2 * p.I : p.H) +
                              (f1 ? fc1_row(wr, p.I, p.fc1_chunked) : wr);
            const float bias = bsrc ? bf16_at(bsrc, wi) : 0.f;
            // Q8: the row's float32 scale (the accumulator holds sum_k q x)
            const float scale = Q8 ? (f1 ? p.s1 : p.s2)[wi] : 1.f;
#pragma unroll 1
            for (int c = 0; c < d.nrows; c += 16) {
                uint32_t v[16];
                tmem_ld_32x32b_x16(tb + c, v);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int n = c + i;
                    const float x = Q8 ? fmaf(f32(v[i]), scale, bias) : f32(v[i]) + bias;
                    if (f1) {
                        const float up = __shfl_xor_sync(0xffffffffu, x, 1);
                        if (!(lane & 1) && n < d.nrows)
                            p.act[static_cast<size_t>(d.row0 + n) * p.I + (wr >> 1)] =
                                __float2bfloat16_rn(swiglu_attr(x, up, p.act_attr));
                    } else if (n < d.nrows) {
                        p.y[static_cast<size_t>(d.row0 + n) * p.H + wr] = __float2bfloat16_rn(x);
                    }
                }
            }
            tc_fence_before();
            if (f1) fence_proxy_async_global();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(smem_u32(&tempty[acc]));
                __threadfence();
                atomicAdd(f1 ? &p.done[d.chunk] : p.fc2_done, 1);
            }
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
        if (p.out != nullptr) {
            // ------------------------------------------------------------ combine
            bool ok = true;
            if (lane == 0) ok = wait_count(p.fc2_done, 4 * (U - U1), abort_flag);
            if (__shfl_sync(0xffffffffu, ok, 0)) {
                const int nvec = p.H / 8;
                const long long total = static_cast<long long>(p.T) * nvec;
                const int et = (warp - 2) * 32 + lane;   // 0..127
                for (long long q = static_cast<long long>(blockIdx.x) * 128 + et; q < total;
                     q += static_cast<long long>(gridDim.x) * 128) {
                    const int t = static_cast<int>(q / nvec), v = static_cast<int>(q - static_cast<long long>(t) * nvec);
                    reinterpret_cast<uint4*>(p.out)[q] =
                        combine_vec_bf16(reinterpret_cast<const uint4*>(p.y), nvec,
                                         ROUTE ? s_pdst : p.perm_dst, ROUTE ? s_rw : p.topk_w,
                                         t, p.k, v, p.rows);
                }
            }
        }
    } else if constexpr (Q8) {
        // the unit sequence, as the other roles read it
        int slot = 0;
        uint32_t uphase = 0;
        auto next_unit = [&]() -> int {
            const bool got = mbar_wait(smem_u32(&ufull[slot]), uphase, abort_flag, kWaitLimitNs);
            const int u = got ? s_unit[slot] : U;
            __syncwarp();
            if (got && lane == 0) mbar_arrive(smem_u32(&uempty[slot]));
            if (++slot == kUnitRing) {
                slot = 0;
                uphase ^= 1u;
            }
            return u;
        };
        if (warp == 6) {
            // -------------------------------------------------------- int8 producer
            // It claims the units: its ring is the deepest (kQStages tiles), so the int8
            // stream runs ahead across unit boundaries instead of waiting for the token
            // producer, which can run only kSlots k-steps ahead of the MMA.
            int claims = 0;
            auto claim_unit = [&]() -> int {
                int u = U;
                if (lane == 0) {
                    if (mbar_wait(smem_u32(&uempty[slot]), uphase ^ 1u, abort_flag, kWaitLimitNs))
                        u = *abort_flag ? U
                            : claims++ == 0 ? static_cast<int>(blockIdx.x)
                                            : static_cast<int>(gridDim.x) + atomicAdd(p.sched, 1);
                    s_unit[slot] = u;
                    mbar_arrive(smem_u32(&ufull[slot]));
                }
                u = __shfl_sync(0xffffffffu, u, 0);
                if (++slot == kUnitRing) {
                    slot = 0;
                    uphase ^= 1u;
                }
                return u;
            };
            int qs = 0;
            uint32_t qphase = 0;
            long long qissued = 0;
            for (;;) {
                const int u = claim_unit();
                if (u >= U) break;
                const DUnit d = decode_dunit(u, U1, MT1, MT2, G, s_off, s_pre);
                const bool f1 = d.phase == 1;
                const int nk = f1 ? nk1 : nk2;
                const CUtensorMap* ma = f1 ? &tmW1 : &tmW2;   // one load site, map chosen at run time
                bool ok = true;
                if (lane == 0) {
                    for (int kb = 0; kb < nk; ++kb) {
                        ok = mbar_wait(smem_u32(&qempty[qs]), qphase ^ 1u, abort_flag, kWaitLimitNs);
                        if (!ok) break;
                        mbar_arrive_expect_tx(smem_u32(&qfull[qs]), kQBytes);
                        tma_load_4d(smem_u32(sQ + qs * kQBytes), ma, smem_u32(&qfull[qs]), kb * BK, 0,
                                    d.mt * (BM / 2), d.g);
                        ++qissued;
                        if (++qs == C::kQStages) {
                            qs = 0;
                            qphase ^= 1u;
                        }
                    }
                }
                if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            }
            if (lane == 0 && *abort_flag) {
                // let the int8 tiles in flight land before the CTA exits
                int dummy = 0;
                for (int s2 = 0; s2 < C::kQStages; ++s2) {
                    if (qissued <= s2) break;
                    const long long fills = (qissued - 1 - s2) / C::kQStages + 1;
                    mbar_wait(smem_u32(&qfull[s2]), static_cast<uint32_t>((fills - 1) & 1), &dummy,
                              kWaitLimitNs / 4);
                }
            }
        } else {
            // -------------------------------------------------------- int8 -> bf16
            // Group grp (warps 7-10, 11-14) converts the stages n with n % 2 == grp (n
            // counts every stage of the launch, as the rings do).  A warp owns the tensor
            // memory lane quadrant warp % 4, i.e. weight rows 32 quad .. 32 quad + 31, one
            // row per lane: for each 64-K slot of the stage the lane reads its row's 64
            // int8 (the tile lands with the 64-byte swizzle, logical 16-byte chunk c of
            // row r at chunk c ^ ((r >> 1) & 3), so a warp's 32 rows read without bank
            // conflicts), converts them to bf16 and writes the 32 packed pairs into the
            // slot's A columns in tensor memory with one tcgen05.st.
            // int8 b -> float32 exactly: the bit pattern 0x4B000000 | (b ^ 0x80) is
            // 2^23 + 128 + b; subtracting 2^23 + 128 leaves b, whose float32 bits end in
            // 16 zero bits (|b| <= 128 has at most 8 significant bits), so its top half
            // is b in bf16.
            const int quad = warp & 3, grp = (warp - 7) >> 2;
            const int row = quad * 32 + lane;
            const uint32_t a_lane = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                                    static_cast<uint32_t>(C::kTmemA);
            int qs = 0, stage = 0, n = 0;
            uint32_t qphase = 0, phase = 0;
            auto next_q = [&]() {
                if (++qs == C::kQStages) {
                    qs = 0;
                    qphase ^= 1u;
                }
            };
            for (;;) {
                const int u = next_unit();
                if (u >= U) break;
                const DUnit d = decode_dunit(u, U1, MT1, MT2, G, s_off, s_pre);
                const int nk = d.phase == 1 ? nk1 : nk2;
                bool ok = true;
                for (int kb0 = 0; kb0 < nk; kb0 += C::kSub, ++n) {
                    const int ns = min(C::kSub, nk - kb0);
                    if ((n & 1) == grp) {
                        if (lane == 0)
                            ok = mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag, kWaitLimitNs);
                        // the whole warp leaves together (lane 0 alone saw the wait give up)
                        ok = __shfl_sync(0xffffffffu, ok, 0);
                        if (!ok) break;
                        tc_fence_after();   // the MMAs that read this stage's A slots have completed
                        const int qs0 = qs;
                        for (int j = 0; j < ns; ++j) {
                            if (lane == 0) ok = mbar_wait(smem_u32(&qfull[qs]), qphase, abort_flag, kWaitLimitNs);
                            ok = __shfl_sync(0xffffffffu, ok, 0);
                            if (!ok) break;
                            const uint8_t* q = sQ + qs * kQBytes + row * BK;
                            uint32_t h[32];
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                const uint4 w = *reinterpret_cast<const uint4*>(q + ((c ^ ((row >> 1) & 3)) << 4));
                                const uint32_t wb[4] = {w.x ^ 0x80808080u, w.y ^ 0x80808080u,
                                                        w.z ^ 0x80808080u, w.w ^ 0x80808080u};
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    // bytes (0, 1) and (2, 3), two float32 subtractions per
                                    // packed add.rn.f32x2 (exact: the differences are integers)
                                    const uint32_t lo = sub_magic_f32x2(
                                        __byte_perm(wb[i], 0x4B000000u, 0x7540u),
                                        __byte_perm(wb[i], 0x4B000000u, 0x7541u));
                                    const uint32_t hi = sub_magic_f32x2(
                                        __byte_perm(wb[i], 0x4B000000u, 0x7542u),
                                        __byte_perm(wb[i], 0x4B000000u, 0x7543u));
                                    h[c * 8 + 2 * i] = lo;
                                    h[c * 8 + 2 * i + 1] = hi;
                                }
                            }
                            tmem_st_32x32b_x32(a_lane + static_cast<uint32_t>((stage * C::kSub + j) * 32), h);
                            next_q();
                        }
                        tmem_wait_st();   // also on a failed wait: no store outlives the warp
                        if (!ok) break;
                        tc_fence_before();   // ... before the MMA thread learns of it
                        __syncwarp();
                        if (lane == 0) {
                            for (int j = 0; j < ns; ++j)
                                mbar_arrive(smem_u32(&qempty[(qs0 + j) % C::kQStages]));
                            mbar_arrive(smem_u32(&full[stage]));
                        }
                    } else {
                        // the other group's stage: only the rings advance
                        for (int j = 0; j < ns; ++j) next_q();
                    }
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
            }
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


// ------------------------------------------------------------------------ host side

// Grid of a persistent decode FFN launch: every unit of both GEMMs, at most one CTA per SM.
int decode_grid(int rows, int E, int H, int I) {
    const long long units =
        (static_cast<long long>((rows + kTokChunk - 1) / kTokChunk) + E) * (2 * I / BM + H / BM);
    const int sms = device_sm_count();
    return static_cast<int>(units < sms ? units : sms);
}

template <bool GATHER, bool ROUTE, bool Q8 = false>
cudaError_t launch_decode(const CUtensorMap& w1, const CUtensorMap& x, const CUtensorMap& w2,
                          const CUtensorMap& a, const DecodeParams& p, int grid, cudaStream_t s) {
    using C = DecodeCfg<Q8>;
    constexpr int kSmem = C::kSmemBytes + (ROUTE ? kRouteSmemBytes : 0);
    static_assert(kSmem <= 227 * 1024, "shared memory");
    auto kern = tc_ffn_decode_kernel<GATHER, ROUTE, Q8>;
    static bool attr_set[64] = {false};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    if (grid <= 0) return cudaSuccess;
    // ROUTE: the routing's grid barrier needs every CTA resident at once, which a
    // cooperative launch guarantees (or refuses: too large a grid is an error, not a wait)
    return launch_k_coop(kern, dim3(grid), dim3(C::kThreads), kSmem, s, ROUTE, w1, x, w2, a, p);
}

}  // namespace

bool tc_ffn_supported(int H, int I) { return H % 64 == 0 && I % 64 == 0 && H > 0 && I > 0; }

bool decode_ffn_supported(int rows, int E, int H, int I) {
    return tc_ffn_supported(H, I) && (2 * I) % BM == 0 && H % BM == 0 &&
           static_cast<long long>(rows) <= static_cast<long long>(kTokChunk) * E;
}

// one completion counter per chunk, the unit scheduler's counter, the fc2 count, the
// routing barrier
int decode_ffn_counters(int rows, int E) { return (rows + kTokChunk - 1) / kTokChunk + E + 3; }

bool fused_route_supported(int T, int H, int E, int k, int I) {
    return T >= 1 && T <= kFusedRouteMaxT && T * k <= kFusedRouteMaxRows && k >= 1 && k <= 32 &&
           k <= E && E <= kMaxExperts && decode_ffn_supported(T * k, E, H, I);
}

cudaError_t launch_ffn_decode(const void* tokens, const int32_t* perm_src, int T,
                              const int32_t* offsets, const void* fc1, const void* fc2, int rows,
                              int H, int E, int I, void* act, void* y, int32_t* done, int32_t* err,
                              const int32_t* perm_dst, const float* topk_w, int k, void* out,
                              cudaStream_t s, const FfnAttrs& ep) {
    if (rows <= 0) return cudaSuccess;
    CUtensorMap w1, x, w2, a;
    const bool q8 = ep.q8();
    if (!tmap::fc1_pairs(&w1, fc1, E, I, H, BM / 2, ep.fc1_chunked, q8)) return cudaErrorInvalidValue;
    if (perm_src) {
        if (!tmap::matrix(&x, tokens, T, H, 1)) return cudaErrorInvalidValue;
    } else {
        if (!tmap::matrix(&x, tokens, rows, H, kBoxTok)) return cudaErrorInvalidValue;
    }
    if (!tmap::plain_pairs(&w2, fc2, E, H, I, BM / 2, q8)) return cudaErrorInvalidValue;
    if (!tmap::matrix(&a, act, rows, I, kBoxTok)) return cudaErrorInvalidValue;
    const int nctr = decode_ffn_counters(rows, E);
    DecodeParams p{};
    p.offsets = offsets;
    p.perm_src = perm_src;
    p.E = E;
    p.rows = rows;
    p.T = T;
    p.H = H;
    p.I = I;
    p.act = static_cast<__nv_bfloat16*>(act);
    p.y = static_cast<__nv_bfloat16*>(y);
    p.done = done;
    p.sched = done + nctr - 3;
    p.fc2_done = done + nctr - 2;
    p.perm_dst = perm_dst;
    p.topk_w = topk_w;
    p.k = k;
    p.out = static_cast<__nv_bfloat16*>(out);
    p.err = err;
    p.act_attr = ep.act;
    p.b1 = static_cast<const __nv_bfloat16*>(ep.fc1_bias);
    p.fc1_chunked = ep.fc1_chunked;
    p.b2 = static_cast<const __nv_bfloat16*>(ep.fc2_bias);
    p.s1 = ep.fc1_scale;
    p.s2 = ep.fc2_scale;
    const int grid = decode_grid(rows, E, H, I);
    if (q8)
        return perm_src ? launch_decode<true, false, true>(w1, x, w2, a, p, grid, s)
                        : launch_decode<false, false, true>(w1, x, w2, a, p, grid, s);
    return perm_src ? launch_decode<true, false>(w1, x, w2, a, p, grid, s)
                    : launch_decode<false, false>(w1, x, w2, a, p, grid, s);
}

namespace {
std::atomic<int> g_route_timeout_test{0};
}  // namespace

void arm_route_timeout_test() { g_route_timeout_test.store(1); }
bool take_route_timeout_test() { return g_route_timeout_test.exchange(0) != 0; }

cudaError_t launch_ffn_decode_routed(const DecodeRoutedArgs& r, cudaStream_t s) {
    const int rows = r.T * r.k;
    if (rows <= 0) return cudaSuccess;
    if (!fused_route_supported(r.T, r.H, r.E, r.k, r.I)) return cudaErrorInvalidValue;
    const bool q8 = r.ep.q8();
    CUtensorMap w1, x, w2, a;
    if (!tmap::fc1_pairs(&w1, r.fc1, r.E, r.I, r.H, BM / 2, r.ep.fc1_chunked, q8))
        return cudaErrorInvalidValue;
    if (!tmap::matrix(&x, r.hidden, r.T, r.H, 1)) return cudaErrorInvalidValue;
    if (!tmap::plain_pairs(&w2, r.fc2, r.E, r.H, r.I, BM / 2, q8)) return cudaErrorInvalidValue;
    if (!tmap::matrix(&a, r.act, rows, r.I, kBoxTok)) return cudaErrorInvalidValue;
    const int nctr = decode_ffn_counters(rows, r.E);
    DecodeParams p{};
    p.E = r.E;
    p.rows = rows;
    p.T = r.T;
    p.H = r.H;
    p.I = r.I;
    p.act = static_cast<__nv_bfloat16*>(r.act);
    p.y = static_cast<__nv_bfloat16*>(r.y);
    p.done = r.counters;
    p.sched = r.counters + nctr - 3;
    p.fc2_done = r.counters + nctr - 2;
    p.route_bar = r.counters + nctr - 1;
    // a timeout armed for testing: one arrival more than the grid gives, a 1 ms limit
    const bool timeout_test = take_route_timeout_test();
    p.route_bar_extra = timeout_test ? 1 : 0;
    p.route_wait_ns = timeout_test ? 1000000ull : kWaitLimitNs;
    p.k = r.k;
    p.out = static_cast<__nv_bfloat16*>(r.out);
    p.err = r.err;
    p.act_attr = r.ep.act;
    p.b1 = static_cast<const __nv_bfloat16*>(r.ep.fc1_bias);
    p.fc1_chunked = r.ep.fc1_chunked;
    p.b2 = static_cast<const __nv_bfloat16*>(r.ep.fc2_bias);
    p.s1 = r.ep.fc1_scale;
    p.s2 = r.ep.fc2_scale;
    p.hidden = r.hidden;
    p.router_w = r.router_w;
    p.bias = r.bias;
    p.normalize = r.normalize ? 1 : 0;
    p.logits = r.logits;
    p.r_topk_idx = r.topk_idx;
    p.r_topk_w = r.topk_w;
    p.r_near_tie = r.near_tie;
    p.r_counts = r.counts;
    p.r_offsets = r.offsets;
    p.r_perm_src = r.perm_src;
    p.r_perm_dst = r.perm_dst;
    const int grid = decode_grid(rows, r.E, r.H, r.I);
    return q8 ? launch_decode<true, true, true>(w1, x, w2, a, p, grid, s)
              : launch_decode<true, true>(w1, x, w2, a, p, grid, s);
}

}  // namespace moe
