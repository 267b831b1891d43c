// Grouped expert GEMMs for large batches on CTA pairs (tcgen05 cta_group::2, sm_100a).
//
// The grouped matmul of grouped_mm_experts_forward ("Contributing Gemma 4 support
// and ONNX export optimizations", "Key Technical Contributions") over each expert's
// contiguous block of permuted rows, with standard SwiGLU on the interleaved fc1
// ("Gemma 4 MoE: re-enable fused com.microsoft::MoE op - #326", "Attribute set"):
//   fc1 + SwiGLU: act[r, i] = swiglu(x[r] . fc1[e, 2i] + b1[e, 2i], x[r] . fc1[e, 2i+1] + b1[e, 2i+1])
//   fc2:          y[r, h]   = act[r] . fc2[e, h] + b2[e, h]
// (standard SwiGLU silu(g) * u, or the op's alpha/beta/limit attributes; the biases
// optional)
//
// Orientation: the expert's WEIGHT rows are the MMA's M side and its tokens the N
// side.  A unit is (expert, tile of up to 256 tokens, tile of 256 weight rows); a
// cluster of two CTAs runs it as one M = 256 MMA: each CTA loads its own 128 weight
// rows and half of the tokens, and accumulates its 128 weight rows x all the tokens
// in its tensor memory.  Per CTA and 64-wide K slice that is 32 KB from L2 for
// 128 x 256 x 64 multiply-adds -- two thirds of what a single-CTA 128 x 256 tile
// needs -- and the token side rounds up to 32 rows, not to a 128-row tile.
//
// Both GEMMs read contiguous token rows (x_perm, act) in one 128-row TMA box.  The
// accumulator holds weight rows x tokens; the weight rows are loaded in fragment order
// (a 5-D view: lane 8 q + j of each 32-lane quadrant holds the quadrant's weight row
// 4 j + q), so that the 16x256b accumulator fragments give a thread four consecutive
// weight rows of two tokens, and every token's outputs leave straight from registers
// (fc2: 8 bytes of one token row per store, fc1 + SwiGLU: 4), a warp's store covering
// four tokens x 64 (32) contiguous bytes, whole 32-byte sectors.
//
// Per CTA, 10 warps:
//   warp 0     TMA producer (both CTAs): its CTA's weight and token slices into a
//              ring of six 64-K slots, signalled in stages of two; completion counted on
//              the even CTA's barrier;
//   warp 1     MMA issuer (even CTA only): tcgen05.mma.cta_group::2 into one of two
//              accumulators; commits free the ring stage in both CTAs and publish
//              the accumulator to both epilogues;
//   warps 2-9  epilogue (both CTAs): tcgen05.ld (16x256b) of their 128 weight rows
//              x the tokens, SwiGLU (fc1) or plain (fc2), stores of token rows from
//              registers, then release the accumulator on the even CTA's barrier.
// Units are statically strided over the pairs (both CTAs walk the same list), so no
// cluster ever waits on another.  Every wait is bounded (2 s) and reports
// MOE_DEVERR_TIMEOUT; both CTAs always reach the final cluster barrier.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tile_map.cuh"
#include "tmap.cuh"

namespace moe {
namespace {

using namespace sm100;

constexpr int kPThreads = 320;                // producer, MMA, 8 epilogue warps
constexpr int kPWRows = 128;                  // weight rows per CTA (256 per pair)
constexpr int kPBK = 64;                      // K per stage: one 128-byte row of bf16
static_assert(kPBK == tmap::kBoxK, "TMA box width");
constexpr int kPTok = 256;                    // tokens per pair tile (<= 128 per CTA)
constexpr int kPStages = 6;                   // 64-K slots in the ring
// The barriers work on stages of kPSub consecutive slots: the MMA thread waits and
// commits once per 128 K.  A wait costs the issuing thread ~160 cycles even on a
// completed phase and a commit ~90, so with one stage per 64 K the four M = 256,
// N = 256 MMAs of a slot (~515 cycles of tensor work) took ~610 cycles; with 128-K
// stages they run back to back (measured stand-alone on a ring of six slots).
constexpr int kPSub = 2;
constexpr int kPBars = kPStages / kPSub;
static_assert(kPBars * kPSub == kPStages, "whole stages");
constexpr int kPABytes = kPWRows * kPBK * 2;  // 16 KB
constexpr int kPBBytes = (kPTok / 2) * kPBK * 2;   // 16 KB
constexpr int kPStageBytes = kPABytes + kPBBytes;
constexpr int kPAccCols = 256;                // one accumulator: 256 fp32 columns
constexpr int kPTmemCols = 512;
constexpr int kPBox = kPTok / 2;              // token rows per TMA box: a CTA's whole half
constexpr uint64_t kPWaitNs = 2000000000ull;
constexpr int kPMiscBytes =
    (2 * kPStages + 4) * 8 + 16 + 2 * (kMaxExperts + 1) * 4 + 64;
constexpr int kPSmemBytes = 1024 + kPStages * kPStageBytes + kPMiscBytes;
static_assert(kPSmemBytes <= 227 * 1024, "shared memory");

struct PairParams {
    const int32_t* offsets;   // [E+1] device
    int E;
    int rows;                 // permuted rows (T k)
    int K;                    // reduction length (multiple of 64)
    int n_out;                // weight rows per expert (2I or H)
    __nv_bfloat16* out;       // [rows, ldo]
    int ldo;                  // I (fc1) or H (fc2)
    int32_t* err;
    SwigluAttr act;           // fc1: SwiGLU attributes
    const __nv_bfloat16* bias;   // [E, n_out] bias of the weight rows, or nullptr
    bool fc1_chunked;            // fc1 (SWIGLU): weights and bias in the chunked layout
};

struct PUnit {
    int g, row0, nrows, n, mt;   // expert, first token row, valid tokens, MMA N, weight tile
};

__device__ __forceinline__ PUnit pair_unit(int u, int MT, int G, const int* s_off, const int* s_pre) {
    PUnit d;
    const int tile = u / MT;
    d.mt = u - tile * MT;
    d.g = tile_group(tile, G, s_pre);
    d.row0 = s_off[d.g] + (tile - s_pre[d.g]) * kPTok;
    d.nrows = min(kPTok, s_off[d.g + 1] - d.row0);
    d.n = ((d.nrows + 31) / 32) * 32;   // each CTA's half: a multiple of 16 rows (TMA boxes)
    return d;
}

template <bool SWIGLU>
__global__ void __launch_bounds__(kPThreads, 1)
tc_pair_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
               const PairParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + kPStages * kPABytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(sB + kPStages * kPBBytes);
    uint64_t* empty = full + kPStages;
    uint64_t* tfull = empty + kPStages;
    uint64_t* tempty = tfull + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* s_off = reinterpret_cast<int*>(tmem_slot + 4);
    int* s_pre = s_off + (kMaxExperts + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool lead = rank == 0;
    const int G = p.E;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPBars; ++s) {
            mbar_init(smem_u32(&full[s]), 1);    // the even CTA's producer (expect_tx)
            mbar_init(smem_u32(&empty[s]), 1);   // the pair MMA's commit
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tfull[a]), 1);
            mbar_init(smem_u32(&tempty[a]), 16); // 8 epilogue warps x 2 CTAs
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmW);
        tma_prefetch_desc(&tmX);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(tmem_slot), kPTmemCols);
        tmem_relinquish_pair();
    }
    // the prologue above touches no global memory; everything below may
    pdl_wait();
    pdl_trigger();
    if (warp == 2) build_group_tiles(p.offsets, p.rows, p.err, G, kPTok, s_off, s_pre, lane);
    tc_fence_before();
    __syncthreads();
    cluster_sync();   // both CTAs' barriers and tensor memory exist before any signal
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int MT = (p.n_out + 2 * kPWRows - 1) / (2 * kPWRows);
    const int num_units = s_pre[G] * MT;
    const int pair = static_cast<int>(blockIdx.x >> 1), npairs = static_cast<int>(gridDim.x >> 1);
    const int nk = p.K / kPBK;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        int stage = 0;
        uint32_t phase = 0;
        for (int u = pair; u < num_units && !*abort_flag; u += npairs) {
            const PUnit d = pair_unit(u, MT, G, s_off, s_pre);
            const int half = d.n / 2;                     // token rows of this CTA
            const int trow0 = d.row0 + static_cast<int>(rank) * half;
            // first weight row of this CTA inside the expert (fc1: in interleaved order),
            // loaded in fragment order through the 5-D view of the weight tensor: plain
            // rows (k, j, q, Q, e) at (k, 0, 0, w_in / 32, g), chunked fc1 (k, j, s, qq, X)
            // at (k, 0, 0, 0, g I / 8 + w_in / 32)
            const int w_in = d.mt * 2 * kPWRows + static_cast<int>(rank) * kPWRows;
            const bool chunked = SWIGLU && p.fc1_chunked;
            const int wc3 = chunked ? 0 : w_in / 32;
            const int wc4 = chunked ? d.g * (p.n_out / 16) + w_in / 32 : d.g;
            // one box of 128 weight rows and one of 128 token rows per CTA (rows past
            // the tile are loaded too, and ignored: one TMA instruction each)
            const uint32_t bytes = static_cast<uint32_t>(2 * kPStageBytes);
            bool ok = true;
            for (int kb0 = 0; kb0 < nk; kb0 += kPSub) {
                const int ns = min(kPSub, nk - kb0);   // slots of this stage (the last may be short)
                if (lane == 0) {
                    ok = mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag, kPWaitNs);
                    if (ok && lead) mbar_arrive_expect_tx(smem_u32(&full[stage]), static_cast<uint32_t>(ns) * bytes);
                }
                // the whole warp leaves together (lane 0 alone saw the wait give up)
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);   // the even CTA's
                if (lane == 0) {
                    for (int j = 0; j < ns; ++j) {
                        const int sl = stage * kPSub + j, kb = kb0 + j;
                        tma_load_5d_pair(smem_u32(sA + sl * kPABytes), &tmW, fb, kb * kPBK, 0, 0, wc3, wc4);
                        tma_load_2d_pair(smem_u32(sB + sl * kPBBytes), &tmX, fb, kb * kPBK, trow0);
                    }
                }
                if (++stage == kPBars) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lead && lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            for (int u = pair; u < num_units && !*abort_flag; u += npairs) {
                const PUnit d = pair_unit(u, MT, G, s_off, s_pre);
                const uint32_t idesc = idesc_bf16_f32(2 * kPWRows, d.n);
                if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1u, abort_flag, kPWaitNs)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kPAccCols);
                bool ok = true;
                for (int kb0 = 0; kb0 < nk; kb0 += kPSub) {
                    const int ns = min(kPSub, nk - kb0);
                    if (!mbar_wait(smem_u32(&full[stage]), phase, abort_flag, kPWaitNs)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    for (int j = 0; j < ns; ++j) {
                        const int sl = stage * kPSub + j, kb = kb0 + j;
                        const uint32_t a0 = smem_u32(sA + sl * kPABytes);
                        const uint32_t b0 = smem_u32(sB + sl * kPBBytes);
#pragma unroll
                        for (int kk = 0; kk < kPBK / 16; ++kk)
                            umma_bf16_pair(d_tmem, smem_desc_sw128(a0 + kk * 32),
                                           smem_desc_sw128(b0 + kk * 32), idesc, (kb | kk) != 0);
                    }
                    umma_commit_pair(smem_u32(&empty[stage]), 0x3);
                    if (++stage == kPBars) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit_pair(smem_u32(&tfull[acc]), 0x3);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // warps 2..9: TMEM lane quadrant warp % 4 (hardware rule), and every other
        // 32-token chunk of the tile.  Thread (fj, ft) = (lane / 4, lane % 4) of the
        // 16x256b fragments holds lanes fj, fj + 8 (first load) and fj + 16, fj + 24
        // (second) of the quadrant -- its weight rows 4 fj .. 4 fj + 3 in fragment
        // order -- for tokens 8 m + 2 ft + e of the chunk (m = 0..3, e = 0, 1).
        const int quad = warp & 3;
        const int part = (warp - 2) >> 2;
        const int fj = lane >> 2, ft = lane & 3;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int u = pair; u < num_units && !*abort_flag; u += npairs) {
            const PUnit d = pair_unit(u, MT, G, s_off, s_pre);
            if (!mbar_wait(smem_u32(&tfull[acc]), acc_phase, abort_flag, kPWaitNs)) break;
            tc_fence_after();
            const uint32_t tb = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                                static_cast<uint32_t>(acc * kPAccCols);
            // this warp's 32 weight rows inside the expert: w0 .. w0+31 (all valid or none:
            // n_out is a multiple of 32); this thread's: wr .. wr + 3 (fc1: interleaved,
            // i.e. gate and up of outputs wr / 2 and wr / 2 + 1)
            const int w0 = d.mt * 2 * kPWRows + static_cast<int>(rank) * kPWRows + quad * 32;
            const bool wvalid = w0 < p.n_out;
            const int wr = w0 + 4 * fj;
            float bias[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                // fc1: the bias of interleaved row wr + q in fc1's layout; fc2: of h
                const int brow = SWIGLU ? fc1_row(wr + q, p.n_out / 2, p.fc1_chunked) : wr + q;
                bias[q] = (p.bias && wvalid)
                              ? bf16_at(p.bias, static_cast<size_t>(d.g) * p.n_out + brow)
                              : 0.f;
            }
#pragma unroll 1
            for (int c = part * 32; c < d.nrows; c += 64) {
                uint32_t lo[16], hi[16];
                tmem_ld_16x256b_x4(tb + c, lo);                  // rows 4 fj, 4 fj + 1
                tmem_ld_16x256b_x4(tb + (16u << 16) + c, hi);    // rows 4 fj + 2, 4 fj + 3
                tmem_wait_ld();
                if (!wvalid) continue;
#pragma unroll
                for (int m = 0; m < 4; ++m) {
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int tok = c + 8 * m + 2 * ft + e;
                        const float x0 = __uint_as_float(lo[4 * m + e]) + bias[0];
                        const float x1 = __uint_as_float(lo[4 * m + 2 + e]) + bias[1];
                        const float x2 = __uint_as_float(hi[4 * m + e]) + bias[2];
                        const float x3 = __uint_as_float(hi[4 * m + 2 + e]) + bias[3];
                        if (tok < d.nrows) {
                            __nv_bfloat16* orow = p.out + static_cast<size_t>(d.row0 + tok) * p.ldo;
                            if constexpr (SWIGLU)
                                *reinterpret_cast<uint32_t*>(orow + (wr >> 1)) =
                                    pack_bf16x2(swiglu_attr_fast(x0, x1, p.act),
                                                swiglu_attr_fast(x2, x3, p.act));
                            else
                                *reinterpret_cast<uint2*>(orow + wr) =
                                    make_uint2(pack_bf16x2(x0, x1), pack_bf16x2(x2, x3));
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
    }

    if (*abort_flag) {
        // copies already issued may still land: give them time before the pair exits
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 200000ull) __nanosleep(1000);
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();   // no CTA leaves while its partner may still read its memory
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kPTmemCols);
    }
    if (threadIdx.x == 0 && *abort_flag && p.err) atomicOr(p.err, kErrTimeout);
}

// ------------------------------------------------------------------------ host side

template <bool SWIGLU>
cudaError_t launch_pair(const CUtensorMap& w, const CUtensorMap& x, const PairParams& p,
                        long long units, cudaStream_t s) {
    auto kern = tc_pair_kernel<SWIGLU>;
    // once per device (outside any stream capture: the first call of every path runs
    // eagerly before a graph is captured): the shared-memory limit and the number of
    // pairs that fit on the GPU at once
    static int max_pairs[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kPThreads);
    cfg.dynamicSmemBytes = kPSmemBytes;
    cfg.stream = s;
    cfg.attrs = attr;
    if (max_pairs[dev] == 0) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kPSmemBytes);
        if (e != cudaSuccess) return e;
        cfg.gridDim = dim3(2 * (device_sm_count() / 2));
        cfg.numAttrs = 1;
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
        if (e != cudaSuccess) return e;
        max_pairs[dev] = n > 0 ? n : 1;
    }
    long long pairs = units < max_pairs[dev] ? units : max_pairs[dev];
    if (pairs <= 0) return cudaSuccess;
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
    cfg.numAttrs = 2;
    count_launch();
    return cudaLaunchKernelEx(&cfg, kern, w, x, p);
}

// One grouped GEMM on CTA pairs: out [rows, ldo] from x [rows, K] (contiguous rows of
// the experts' blocks) and the weights w [E, n_out, K] of E experts (both through the
// 5-D fragment-order views, the chunked one reading fc1 in place).
cudaError_t pair_gemm(bool swiglu, const void* x, int rows, int K, const void* w, int E, int n_out,
                      const int32_t* offsets, void* out, int ldo, int32_t* err, cudaStream_t s,
                      const FfnAttrs& at, const void* bias) {
    CUtensorMap mw, mx;
    const bool ok_w = (swiglu && at.fc1_chunked) ? tmap::fc1_quad_rows_chunked(&mw, w, E, n_out / 2, K)
                                                 : tmap::quad_rows(&mw, w, E, n_out, K);
    if (!ok_w) return cudaErrorInvalidValue;
    if (!tmap::matrix(&mx, x, rows, K, kPBox)) return cudaErrorInvalidValue;
    PairParams p{offsets, E, rows, K, n_out, static_cast<__nv_bfloat16*>(out), ldo, err, at.act,
                 static_cast<const __nv_bfloat16*>(bias), at.fc1_chunked};
    const long long units = (static_cast<long long>((rows + kPTok - 1) / kPTok) + E) *
                            ((n_out + 2 * kPWRows - 1) / (2 * kPWRows));
    return swiglu ? launch_pair<true>(mw, mx, p, units, s) : launch_pair<false>(mw, mx, p, units, s);
}

}  // namespace

bool pair_ffn_supported(int H, int I) { return H > 0 && I > 0 && H % 64 == 0 && I % 64 == 0; }

cudaError_t launch_ffn_pair(const void* x_perm, const int32_t* offsets, const void* fc1,
                            const void* fc2, int rows, int H, int E, int I, void* act, void* y,
                            int32_t* err, cudaStream_t s, cudaEvent_t mid, const FfnAttrs& ep) {
    if (rows <= 0) return cudaSuccess;
    cudaError_t e = pair_gemm(true, x_perm, rows, H, fc1, E, 2 * I, offsets, act, I, err, s, ep,
                              ep.fc1_bias);
    if (e != cudaSuccess) return e;
    if (mid) record_event(mid, s);
    return pair_gemm(false, act, rows, I, fc2, E, H, offsets, y, H, err, s, ep, ep.fc2_bias);
}

}  // namespace moe
