// C ABI of the fused MoE FFN layer: argument checks, workspace layout and the
// order of the launches.  Declarations and contracts: include/moe_b200.h.
#include <math.h>
#include <string.h>

#include <atomic>

#include "common.cuh"
#include "kernels.h"
#include "moe_b200.h"

namespace moe {

int device_sm_count() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

namespace {
std::atomic<unsigned long long> g_launches{0};
}  // namespace

void count_launch(int n) { g_launches.fetch_add(static_cast<unsigned long long>(n)); }

void record_event(cudaEvent_t ev, cudaStream_t s) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
        cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal);
    else
        cudaEventRecord(ev, s);
}

namespace {

constexpr size_t kAlign = 256;
constexpr int kNumStageEvents = 6;

cudaEvent_t g_events[kNumStageEvents];
bool g_events_on = false;

size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

struct Carver {
    size_t off = 0;
    size_t take(size_t bytes) {
        const size_t r = off;
        off = align_up(off + bytes);
        return r;
    }
};

struct FwdLayout {
    size_t hdr, logits, idx, w, near, tile_counts, counts, offsets, perm_src, perm_dst, ctr,
        x_perm, act, y, xn, total;
};

size_t elem_size(moe_dtype dt) { return dt == MOE_BF16 ? 2 : 4; }

constexpr int kPathSmallRoute = 1, kPathDecodeFfn = 2, kPathTcRouter = 4, kPathTokenGemm = 8,
              kPathF32Ffn = 16, kPathFusedRoute = 32;

// The bf16 decode FFN gathers its token rows from hidden itself (tile::gather4, four rows
// per load) when each expert has at most 4 rows on average; with more, TMA row gathers
// cannot keep up and the rows are gathered once into x_perm and loaded in 16-row boxes.
bool decode_gathers(int T, int H, int E, int k, int I, moe_dtype dt) {
    const long long rows = static_cast<long long>(T) * k;
    return dt == MOE_BF16 && rows <= 4LL * E && decode_ffn_supported(static_cast<int>(rows), E, H, I);
}

FwdLayout fwd_layout(int T, int H, int E, int k, int I, moe_dtype dt) {
    const size_t es = elem_size(dt);
    const size_t rows = static_cast<size_t>(T) * k;
    const size_t nt = static_cast<size_t>(num_token_tiles(T));
    Carver c;
    FwdLayout L;
    // the header, the decode FFN's counters and the tile counts come first: one memset
    // clears them
    L.hdr = c.take(kAlign);   // [0] error word
    L.ctr = c.take(static_cast<size_t>(decode_ffn_counters(static_cast<int>(rows), E)) * 4);
    L.tile_counts = c.take(nt * E * 4);
    L.logits = c.take(static_cast<size_t>(T) * E * 4);
    L.idx = c.take(rows * 4);
    L.w = c.take(rows * 4);
    L.near = c.take(static_cast<size_t>(T) * 4);
    L.counts = c.take(static_cast<size_t>(E) * 4);
    L.offsets = c.take(static_cast<size_t>(E + 1) * 4);
    L.perm_src = c.take(rows * 4);
    L.perm_dst = c.take(rows * 4);
    // the permuted copy of the token rows, unless the decode FFN gathers them itself
    L.x_perm = c.take(decode_gathers(T, H, E, k, I, dt) ? 0 : rows * H * es);
    L.act = c.take(rows * I * es);
    L.y = c.take(rows * H * es);
    L.xn = c.take(static_cast<size_t>(T) * H * es);   // the normalised input (pre-FFN norm)
    L.total = c.off;
    return L;
}

struct PermLayout {
    size_t hdr, tile_counts, total;
};

PermLayout perm_layout(int T, int E) {
    const size_t nt = static_cast<size_t>(num_token_tiles(T));
    Carver c;
    PermLayout L;
    L.hdr = c.take(kAlign);
    L.tile_counts = c.take(nt * E * 4);
    L.total = c.off;
    return L;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool valid_dtype(moe_dtype dt) { return dt == MOE_F32 || dt == MOE_BF16; }

// Sizes shared by the layer and the staged calls.
bool valid_sizes(int T, int H, int E, int k) {
    if (T < 0 || H <= 0 || E <= 0 || E > kMaxExperts || k < 1 || k > E) return false;
    if (H % 8 != 0) return false;
    if (static_cast<long long>(T) * k > (1LL << 30)) return false;
    return true;
}

bool standard_swiglu(const moe_swiglu& a) {
    return a.alpha == 1.0f && a.beta == 0.0f && isinf(a.limit) && a.limit > 0;
}

// Finite alpha and beta, a positive limit (+inf = no clipping).
bool valid_swiglu(const moe_swiglu& a) {
    return isfinite(a.alpha) && isfinite(a.beta) && !isnan(a.limit) && a.limit > 0.0f;
}

bool valid_layout(moe_fc1_layout l) { return l == MOE_FC1_INTERLEAVED || l == MOE_FC1_CHUNKED; }

bool valid_eps(float eps) { return isfinite(eps) && eps >= 0.0f; }

FfnAttrs make_ffn_attrs(const moe_swiglu& a, moe_fc1_layout layout, const void* fc1_bias,
                        const void* fc2_bias) {
    FfnAttrs ep;
    ep.act = SwigluAttr{a.alpha, a.beta, a.limit, standard_swiglu(a) ? 1 : 0};
    ep.fc1_chunked = layout == MOE_FC1_CHUNKED;
    ep.fc1_bias = fc1_bias;
    ep.fc2_bias = fc2_bias;
    return ep;
}

// Which kernels moe_forward runs for these sizes (bits of moe_forward_path, declared
// above).
// Up to this many tokens a bf16 batch is routed by the split router + one CTA; above
// it, by the tensor-core router with the routing in its epilogue.
constexpr int kRouteSmallTcT = 16;

int forward_path(int T, int H, int E, int k, int I, moe_dtype dt) {
    const bool bf16 = dt == MOE_BF16;
    const int rows = T * k;
    // small bf16 batches: the whole layer in one launch
    if (bf16 && fused_route_supported(T, H, E, k, I)) return kPathFusedRoute | kPathDecodeFfn;
    int path = 0;
    if (bf16 && T > kRouteSmallTcT && tc_route_supported(H, E, k)) path |= kPathTcRouter;
    else if (T <= kRouteSmallMaxT && k <= kRouteSmallMaxK) path |= kPathSmallRoute;
    if (!bf16) path |= kPathF32Ffn;
    else if (decode_ffn_supported(rows, E, H, I)) path |= kPathDecodeFfn;
    else path |= kPathTokenGemm;
    return path;
}

// int8 experts: the decode FFN, with the routing inside its launch for small batches,
// else after the staged routing kernels (0: no such path for these sizes)
int forward_path_q8(int T, int H, int E, int k, int I) {
    const int rows = T * k;
    if (fused_route_supported(T, H, E, k, I)) return kPathFusedRoute | kPathDecodeFfn;
    if (!decode_ffn_supported(rows, E, H, I)) return 0;
    if (T > kRouteSmallTcT && tc_route_supported(H, E, k)) return kPathTcRouter | kPathDecodeFfn;
    if (T <= kRouteSmallMaxT && k <= kRouteSmallMaxK) return kPathSmallRoute | kPathDecodeFfn;
    return kPathDecodeFfn;   // routed by the float32-logit top-k kernels
}

void record(int i, cudaStream_t s) {
    if (g_events_on) record_event(g_events[i], s);
}

#define MOE_CUDA(call)                                  \
    do {                                                \
        if ((call) != cudaSuccess) return MOE_ERR_CUDA; \
    } while (0)

// x_perm from hidden: token by token (each hidden row read once) for k <= 32, else row
// by row through perm_src.
cudaError_t gather_rows(const void* hidden, const int32_t* perm_src, const int32_t* perm_dst,
                        const int32_t* offsets, int T, int E, int k, int H, moe_dtype dt,
                        void* x_perm, cudaStream_t s) {
    const int es = static_cast<int>(elem_size(dt));
    if (k <= 32) return launch_gather_by_token(hidden, perm_dst, T, k, T * k, H, es, x_perm, s);
    return launch_gather(hidden, perm_src, offsets, E, T, T * k, H, es, x_perm, s);
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

int moe_version(void) { return 220; }

void moe_debug_arm_route_barrier_timeout(void) { arm_route_timeout_test(); }

unsigned long long moe_kernel_launches(void) { return g_launches.load(); }

const char* moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
        case MOE_ERR_DEVICE: return "MOE_ERR_DEVICE";
        case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
    }
    return "MOE_ERR_UNKNOWN";
}

size_t moe_workspace_size(int T, int H, int E, int k, int I, moe_dtype dt) {
    if (!valid_sizes(T, H, E, k) || I <= 0 || I % 8 != 0 || !valid_dtype(dt)) return 0;
    return fwd_layout(T, H, E, k, I, dt).total;
}

size_t moe_permute_workspace_size(int T, int E) {
    if (T < 0 || E <= 0 || E > kMaxExperts) return 0;
    return perm_layout(T, E).total;
}

size_t moe_expert_ffn_workspace_size(int rows, int I, moe_dtype dt) {
    if (rows < 0 || I <= 0 || !valid_dtype(dt)) return 0;
    // error word | activations [rows, I] | counters of the decode FFN (E <= 256)
    return kAlign + align_up(static_cast<size_t>(rows) * I * elem_size(dt)) +
           align_up(static_cast<size_t>(decode_ffn_counters(rows, kMaxExperts)) * 4);
}

int moe_forward_path(int T, int H, int E, int k, int I, moe_dtype dt) {
    if (!valid_sizes(T, H, E, k) || I <= 0 || I % 8 || !valid_dtype(dt)) return 0;
    return forward_path(T, H, E, k, I, dt);
}

int32_t* moe_workspace_error_word(void* workspace) { return static_cast<int32_t*>(workspace); }

moe_status moe_set_stage_events(void* const* events, int n_events) {
    if (events == nullptr) {
        g_events_on = false;
        return MOE_OK;
    }
    if (n_events != kNumStageEvents) return MOE_ERR_INVALID_ARG;
    for (int i = 0; i < kNumStageEvents; ++i) {
        if (events[i] == nullptr) return MOE_ERR_INVALID_ARG;
        g_events[i] = static_cast<cudaEvent_t>(events[i]);
    }
    g_events_on = true;
    return MOE_OK;
}

moe_status moe_route(const void* hidden, const void* router_w, const float* router_bias, int T,
                     int H, int E, int k, int normalize, moe_dtype dt, int32_t* topk_idx,
                     float* topk_w, float* logits, int32_t* near_tie, void* stream) {
    if (!valid_sizes(T, H, E, k) || !valid_dtype(dt)) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!hidden || !router_w || !topk_idx || !topk_w || !logits) return MOE_ERR_INVALID_ARG;
    if (!aligned(hidden, 16) || !aligned(router_w, 16) || !aligned(topk_idx, 4) ||
        !aligned(topk_w, 4) || !aligned(logits, 16) || (router_bias && !aligned(router_bias, 4)) ||
        (near_tie && !aligned(near_tie, 4)))
        return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dt == MOE_BF16 && T > kRouteSmallTcT && tc_route_supported(H, E, k))
        return launch_route_tc(hidden, router_w, router_bias, T, H, E, k, normalize, topk_idx,
                               topk_w, near_tie, logits, nullptr, nullptr, s) == cudaSuccess
                   ? MOE_OK
                   : MOE_ERR_CUDA;
    MOE_CUDA(launch_router_logits_simt(hidden, router_w, T, H, E, dt == MOE_BF16, logits, s));
    TopkHistArgs a;
    a.logits = logits;
    a.bias = router_bias;
    a.logits_biased = router_bias ? logits : nullptr;
    a.T = T;
    a.E = E;
    a.k = k;
    a.normalize = normalize ? 1 : 0;
    a.topk_idx = topk_idx;
    a.topk_w = topk_w;
    a.near_tie = near_tie;
    MOE_CUDA(launch_topk_hist(a, s));
    return MOE_OK;
}

moe_status moe_permute(const void* hidden, const int32_t* topk_idx, int T, int H, int E, int k,
                       moe_dtype dt, int32_t* counts, int32_t* offsets, int32_t* perm_src,
                       int32_t* perm_dst, void* x_perm, int32_t* err_word, void* workspace,
                       size_t ws_bytes, void* stream) {
    if (!valid_sizes(T, H, E, k) || !valid_dtype(dt)) return MOE_ERR_INVALID_ARG;
    if (!topk_idx || !counts || !offsets || !perm_src || !perm_dst || !err_word || !workspace)
        return MOE_ERR_INVALID_ARG;
    if ((hidden == nullptr) != (x_perm == nullptr)) return MOE_ERR_INVALID_ARG;
    if ((hidden && !aligned(hidden, 16)) || (x_perm && !aligned(x_perm, 16)) ||
        !aligned(workspace, kAlign))
        return MOE_ERR_INVALID_ARG;
    const PermLayout L = perm_layout(T, E);
    if (ws_bytes < L.total) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char* ws = static_cast<char*>(workspace);
    if (T == 0) {
        MOE_CUDA(cudaMemsetAsync(counts, 0, static_cast<size_t>(E) * 4, s));
        MOE_CUDA(cudaMemsetAsync(offsets, 0, static_cast<size_t>(E + 1) * 4, s));
        return MOE_OK;
    }
    TopkHistArgs a;
    a.T = T;
    a.E = E;
    a.k = k;
    a.topk_idx = const_cast<int32_t*>(topk_idx);
    a.tile_counts = reinterpret_cast<int32_t*>(ws + L.tile_counts);
    a.err = err_word;
    MOE_CUDA(launch_topk_hist(a, s));
    MOE_CUDA(launch_scatter(topk_idx, a.tile_counts, T, E, k, counts, offsets, perm_src, perm_dst,
                            err_word, s));
    if (x_perm)
        MOE_CUDA(launch_gather(hidden, perm_src, offsets, E, T, T * k, H, static_cast<int>(elem_size(dt)),
                               x_perm, s));
    return MOE_OK;
}

moe_status moe_expert_ffn(const void* x_perm, const int32_t* offsets, const void* fc1,
                          const void* fc2, const void* fc1_bias, const void* fc2_bias, int rows,
                          int H, int E, int I, moe_swiglu act, moe_fc1_layout fc1_layout,
                          moe_dtype dt, void* y_perm, void* workspace, size_t ws_bytes,
                          void* stream) {
    if (rows < 0 || H <= 0 || H % 8 || I <= 0 || I % 8 || E <= 0 || E > kMaxExperts ||
        !valid_dtype(dt) || !valid_swiglu(act) || !valid_layout(fc1_layout))
        return MOE_ERR_INVALID_ARG;
    if ((fc1_bias && !aligned(fc1_bias, elem_size(dt))) || (fc2_bias && !aligned(fc2_bias, elem_size(dt))))
        return MOE_ERR_INVALID_ARG;
    if (dt == MOE_BF16 && !tc_ffn_supported(H, I)) return MOE_ERR_UNSUPPORTED;
    if (rows == 0) return MOE_OK;
    if (!x_perm || !offsets || !fc1 || !fc2 || !y_perm || !workspace) return MOE_ERR_INVALID_ARG;
    if (!aligned(x_perm, 16) || !aligned(fc1, 16) || !aligned(fc2, 16) || !aligned(y_perm, 16) ||
        !aligned(workspace, kAlign))
        return MOE_ERR_INVALID_ARG;
    if (ws_bytes < moe_expert_ffn_workspace_size(rows, I, dt)) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char* ws = static_cast<char*>(workspace);
    int32_t* err = reinterpret_cast<int32_t*>(ws);   // scratch error word of this call
    void* act_buf = ws + kAlign;
    int32_t* ctr = reinterpret_cast<int32_t*>(ws + kAlign +
                                              align_up(static_cast<size_t>(rows) * I * elem_size(dt)));
    MOE_CUDA(cudaMemsetAsync(err, 0, 4, s));
    const FfnAttrs ep = make_ffn_attrs(act, fc1_layout, fc1_bias, fc2_bias);
    if (dt == MOE_BF16 && decode_ffn_supported(rows, E, H, I)) {
        MOE_CUDA(cudaMemsetAsync(ctr, 0, static_cast<size_t>(decode_ffn_counters(rows, E)) * 4, s));
        MOE_CUDA(launch_ffn_decode(x_perm, nullptr, rows, offsets, fc1, fc2, rows, H, E, I,
                                   act_buf, y_perm, ctr, err, nullptr, nullptr, 0, nullptr, s, ep));
    } else if (dt == MOE_BF16) {
        MOE_CUDA(launch_ffn_pair(x_perm, offsets, fc1, fc2, rows, H, E, I, act_buf, y_perm, err, s,
                                 nullptr, ep));
    } else {
        MOE_CUDA(launch_ffn_simt_f32(static_cast<const float*>(x_perm), offsets,
                                     static_cast<const float*>(fc1), static_cast<const float*>(fc2),
                                     rows, H, E, I, static_cast<float*>(act_buf),
                                     static_cast<float*>(y_perm), s, nullptr, ep));
    }
    return MOE_OK;
}

moe_status moe_combine(const void* y_perm, const int32_t* perm_dst, const float* topk_w, int T,
                       int H, int k, moe_dtype dt, void* out, void* stream) {
    if (T < 0 || H <= 0 || H % 8 || k < 1 || k > kMaxExperts || !valid_dtype(dt) ||
        static_cast<long long>(T) * k > (1LL << 30))
        return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!y_perm || !perm_dst || !topk_w || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned(y_perm, 16) || !aligned(out, 16)) return MOE_ERR_INVALID_ARG;
    MOE_CUDA(launch_combine(y_perm, perm_dst, topk_w, T, H, k, dt == MOE_BF16, out,
                            static_cast<cudaStream_t>(stream)));
    return MOE_OK;
}

moe_status moe_rmsnorm(const void* x, const void* weight, int T, int H, float eps, moe_dtype dt,
                       void* y, void* stream) {
    if (T < 0 || H <= 0 || H % 8 || !valid_dtype(dt) || !valid_eps(eps)) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !weight || !y || !aligned(x, 16) || !aligned(weight, 16) || !aligned(y, 16))
        return MOE_ERR_INVALID_ARG;
    const size_t bytes = static_cast<size_t>(T) * H * elem_size(dt);
    const uintptr_t a = reinterpret_cast<uintptr_t>(x), b = reinterpret_cast<uintptr_t>(y);
    if (a < b + bytes && b < a + bytes) return MOE_ERR_INVALID_ARG;   // overlap
    MOE_CUDA(launch_rmsnorm(x, weight, T, H, eps, dt == MOE_BF16, y, nullptr, 0,
                            static_cast<cudaStream_t>(stream)));
    return MOE_OK;
}

// The layer; with fc1_scale / fc2_scale, fc1 and fc2 hold int8 weights (moe_forward_q8).
static moe_status forward_impl(const void* hidden, const void* norm_weight, float norm_eps,
                               const void* router_w, const float* router_bias, const void* fc1,
                               const void* fc2, const void* fc1_bias, const void* fc2_bias, int T,
                               int H, int E, int k, int I, int normalize, moe_swiglu act,
                               moe_fc1_layout fc1_layout, moe_dtype dt, void* out, void* workspace,
                               size_t ws_bytes, void* stream, const float* fc1_scale,
                               const float* fc2_scale) {
    if (!valid_sizes(T, H, E, k) || I <= 0 || I % 8 || !valid_dtype(dt) || !valid_swiglu(act) ||
        !valid_layout(fc1_layout) || (norm_weight && !valid_eps(norm_eps)))
        return MOE_ERR_INVALID_ARG;
    const bool q8 = fc1_scale != nullptr;
    if (q8 && (dt != MOE_BF16 || !fc2_scale || !aligned(fc1_scale, 4) || !aligned(fc2_scale, 4)))
        return MOE_ERR_INVALID_ARG;
    if (norm_weight && !aligned(norm_weight, 16)) return MOE_ERR_INVALID_ARG;
    if ((fc1_bias && !aligned(fc1_bias, elem_size(dt))) || (fc2_bias && !aligned(fc2_bias, elem_size(dt))))
        return MOE_ERR_INVALID_ARG;
    if (dt == MOE_BF16 && !tc_ffn_supported(H, I)) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (!hidden || !router_w || !fc1 || !fc2 || !out || !workspace) return MOE_ERR_INVALID_ARG;
    if (!aligned(hidden, 16) || !aligned(router_w, 16) || !aligned(fc1, 16) || !aligned(fc2, 16) ||
        !aligned(out, 16) || !aligned(workspace, kAlign) ||
        (router_bias && !aligned(router_bias, 4)))
        return MOE_ERR_INVALID_ARG;
    const FwdLayout L = fwd_layout(T, H, E, k, I, dt);
    if (ws_bytes < L.total) return MOE_ERR_INVALID_ARG;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char* ws = static_cast<char*>(workspace);
    int32_t* err = reinterpret_cast<int32_t*>(ws + L.hdr);
    float* logits = reinterpret_cast<float*>(ws + L.logits);
    int32_t* idx = reinterpret_cast<int32_t*>(ws + L.idx);
    float* w = reinterpret_cast<float*>(ws + L.w);
    int32_t* offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
    int32_t* perm_src = reinterpret_cast<int32_t*>(ws + L.perm_src);
    int32_t* perm_dst = reinterpret_cast<int32_t*>(ws + L.perm_dst);
    void* x_perm = ws + L.x_perm;
    void* act_buf = ws + L.act;
    void* y = ws + L.y;
    const bool bf16 = dt == MOE_BF16;
    const int rows = T * k;

    int path = forward_path(T, H, E, k, I, dt);
    FfnAttrs ep = make_ffn_attrs(act, fc1_layout, fc1_bias, fc2_bias);
    if (q8) {
        // int8 experts run in the decode FFN only, routed by the staged kernels
        path = forward_path_q8(T, H, E, k, I);
        if (path == 0) return MOE_ERR_UNSUPPORTED;
        ep.fc1_scale = fc1_scale;
        ep.fc2_scale = fc2_scale;
    }
    int32_t* ctr = reinterpret_cast<int32_t*>(ws + L.ctr);
    int32_t* counts = reinterpret_cast<int32_t*>(ws + L.counts);
    int32_t* near = reinterpret_cast<int32_t*>(ws + L.near);
    record(0, s);
    // The first launch zeroes what must start at zero (the error word, the decode-FFN
    // counters, the tile counts; the split router of the small-route path clears the
    // header itself) and, with a norm weight, also writes the normalised input, which
    // then replaces `hidden` everywhere below.
    const size_t clear_end = (path & kPathFusedRoute) ? L.tile_counts
                             : (path & kPathSmallRoute) ? L.hdr : L.logits;
    if (norm_weight) {
        MOE_CUDA(launch_rmsnorm(hidden, norm_weight, T, H, norm_eps, bf16, ws + L.xn, ws + L.hdr,
                                clear_end - L.hdr, s));
        hidden = ws + L.xn;
    } else if (clear_end > L.hdr) {
        MOE_CUDA(launch_clear(ws + L.hdr, clear_end - L.hdr, s));
    }
    if (path & kPathFusedRoute) {
        // one launch: routing, fc1 + SwiGLU, fc2 and the weighted combine
        record(1, s);
        record(2, s);
        DecodeRoutedArgs a{};
        a.hidden = hidden;
        a.router_w = router_w;
        a.bias = router_bias;
        a.fc1 = fc1;
        a.fc2 = fc2;
        a.T = T;
        a.H = H;
        a.E = E;
        a.k = k;
        a.I = I;
        a.normalize = normalize ? 1 : 0;
        a.logits = logits;
        a.topk_idx = idx;
        a.topk_w = w;
        a.near_tie = near;
        a.counts = counts;
        a.offsets = offsets;
        a.perm_src = perm_src;
        a.perm_dst = perm_dst;
        a.act = act_buf;
        a.y = y;
        a.counters = ctr;
        a.err = err;
        a.out = out;
        a.ep = ep;
        MOE_CUDA(launch_ffn_decode_routed(a, s));
        record(3, s);
        record(4, s);
        record(5, s);
        return MOE_OK;
    }
    if (path & kPathSmallRoute) {
        // logits on many CTAs (which also clear the header), then one CTA for top-k,
        // bincount, scan and the stable permutation
        MOE_CUDA(launch_router_logits_split(hidden, router_w, T, H, E, bf16, logits, err, s));
        RouteSmallArgs a;
        a.logits = logits;
        a.bias = router_bias;
        a.T = T;
        a.E = E;
        a.k = k;
        a.normalize = normalize ? 1 : 0;
        a.topk_idx = idx;
        a.topk_w = w;
        a.near_tie = near;
        a.counts = counts;
        a.offsets = offsets;
        a.perm_src = perm_src;
        a.perm_dst = perm_dst;
        if (path & kPathDecodeFfn) {
            a.zero_words = ctr;
            a.n_zero = decode_ffn_counters(rows, E);
        }
        MOE_CUDA(launch_route_small(a, s));
        record(1, s);
    } else {
        int32_t* tile_counts = reinterpret_cast<int32_t*>(ws + L.tile_counts);
        if (path & kPathTcRouter) {
            // logits on the tensor cores, routing and per-tile bincount in the epilogue
            MOE_CUDA(launch_route_tc(hidden, router_w, router_bias, T, H, E, k, normalize, idx, w,
                                     near, nullptr, tile_counts, err, s));
        } else {
            MOE_CUDA(launch_router_logits_simt(hidden, router_w, T, H, E, bf16, logits, s));
            TopkHistArgs a;
            a.logits = logits;
            a.bias = router_bias;
            a.T = T;
            a.E = E;
            a.k = k;
            a.normalize = normalize ? 1 : 0;
            a.topk_idx = idx;
            a.topk_w = w;
            a.near_tie = near;
            a.tile_counts = tile_counts;
            a.err = err;
            MOE_CUDA(launch_topk_hist(a, s));
        }
        record(1, s);
        MOE_CUDA(launch_scatter(idx, tile_counts, T, E, k, counts, offsets, perm_src, perm_dst,
                                err, s));
    }
    if (path & kPathDecodeFfn) {
        // fc1 + SwiGLU and fc2 in one launch.  With at most 4 rows per expert on
        // average, fc1 gathers its token rows straight from hidden (tile::gather4, four
        // rows per load); with more, the rows are gathered once into x_perm and loaded
        // in 16-row boxes.
        const bool tma_gather = decode_gathers(T, H, E, k, I, dt);
        if (!tma_gather)
            MOE_CUDA(gather_rows(hidden, perm_src, perm_dst, offsets, T, E, k, H, dt, x_perm, s));
        record(2, s);
        // ... and the weighted combine, after every fc2 unit has published its rows
        MOE_CUDA(launch_ffn_decode(tma_gather ? hidden : x_perm, tma_gather ? perm_src : nullptr,
                                   T, offsets, fc1, fc2, rows, H, E, I, act_buf, y, ctr, err,
                                   perm_dst, w, k, out, s, ep));
        record(3, s);
        record(4, s);
        record(5, s);
        return MOE_OK;
    } else {
        MOE_CUDA(gather_rows(hidden, perm_src, perm_dst, offsets, T, E, k, H, dt, x_perm, s));
        record(2, s);
        cudaEvent_t mid = g_events_on ? g_events[3] : nullptr;
        if (bf16)
            MOE_CUDA(launch_ffn_pair(x_perm, offsets, fc1, fc2, rows, H, E, I, act_buf, y, err, s,
                                     mid, ep));
        else
            MOE_CUDA(launch_ffn_simt_f32(static_cast<const float*>(x_perm), offsets,
                                         static_cast<const float*>(fc1),
                                         static_cast<const float*>(fc2), rows, H, E, I,
                                         static_cast<float*>(act_buf), static_cast<float*>(y), s,
                                         mid, ep));
    }
    record(4, s);
    MOE_CUDA(launch_combine(y, perm_dst, w, T, H, k, bf16, out, s));
    record(5, s);
    return MOE_OK;
}

moe_status moe_forward(const void* hidden, const void* norm_weight, float norm_eps,
                       const void* router_w, const float* router_bias,
                       const void* fc1, const void* fc2, const void* fc1_bias, const void* fc2_bias,
                       int T, int H, int E, int k, int I, int normalize, moe_swiglu act,
                       moe_fc1_layout fc1_layout, moe_dtype dt, void* out, void* workspace,
                       size_t ws_bytes, void* stream) {
    return forward_impl(hidden, norm_weight, norm_eps, router_w, router_bias, fc1, fc2, fc1_bias,
                        fc2_bias, T, H, E, k, I, normalize, act, fc1_layout, dt, out, workspace,
                        ws_bytes, stream, nullptr, nullptr);
}

moe_status moe_forward_q8(const void* hidden, const void* norm_weight, float norm_eps,
                          const void* router_w, const float* router_bias, const int8_t* fc1_q,
                          const float* fc1_scale, const int8_t* fc2_q, const float* fc2_scale,
                          const void* fc1_bias, const void* fc2_bias, int T, int H, int E, int k,
                          int I, int normalize, moe_swiglu act, moe_fc1_layout fc1_layout,
                          void* out, void* workspace, size_t ws_bytes, void* stream) {
    if (!fc1_scale || !fc2_scale) return MOE_ERR_INVALID_ARG;
    return forward_impl(hidden, norm_weight, norm_eps, router_w, router_bias, fc1_q, fc2_q,
                        fc1_bias, fc2_bias, T, H, E, k, I, normalize, act, fc1_layout, MOE_BF16, out,
                        workspace, ws_bytes, stream, fc1_scale, fc2_scale);
}

moe_status moe_expert_ffn_q8(const void* x_perm, const int32_t* offsets, const int8_t* fc1_q,
                             const float* fc1_scale, const int8_t* fc2_q, const float* fc2_scale,
                             const void* fc1_bias, const void* fc2_bias, int rows, int H, int E,
                             int I, moe_swiglu act, moe_fc1_layout fc1_layout, void* y_perm,
                             void* workspace, size_t ws_bytes, void* stream) {
    if (rows < 0 || H <= 0 || H % 8 || I <= 0 || I % 8 || E <= 0 || E > kMaxExperts ||
        !valid_swiglu(act) || !valid_layout(fc1_layout))
        return MOE_ERR_INVALID_ARG;
    if ((fc1_bias && !aligned(fc1_bias, 2)) || (fc2_bias && !aligned(fc2_bias, 2)))
        return MOE_ERR_INVALID_ARG;
    if (!fc1_scale || !fc2_scale || !aligned(fc1_scale, 4) || !aligned(fc2_scale, 4))
        return MOE_ERR_INVALID_ARG;
    if (!decode_ffn_supported(rows, E, H, I)) return MOE_ERR_UNSUPPORTED;
    if (rows == 0) return MOE_OK;
    if (!x_perm || !offsets || !fc1_q || !fc2_q || !y_perm || !workspace) return MOE_ERR_INVALID_ARG;
    if (!aligned(x_perm, 16) || !aligned(fc1_q, 16) || !aligned(fc2_q, 16) || !aligned(y_perm, 16) ||
        !aligned(workspace, kAlign))
        return MOE_ERR_INVALID_ARG;
    if (ws_bytes < moe_expert_ffn_workspace_size(rows, I, MOE_BF16)) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char* ws = static_cast<char*>(workspace);
    int32_t* err = reinterpret_cast<int32_t*>(ws);
    void* act_buf = ws + kAlign;
    int32_t* ctr = reinterpret_cast<int32_t*>(ws + kAlign + align_up(static_cast<size_t>(rows) * I * 2));
    MOE_CUDA(cudaMemsetAsync(err, 0, 4, s));
    FfnAttrs ep = make_ffn_attrs(act, fc1_layout, fc1_bias, fc2_bias);
    ep.fc1_scale = fc1_scale;
    ep.fc2_scale = fc2_scale;
    MOE_CUDA(cudaMemsetAsync(ctr, 0, static_cast<size_t>(decode_ffn_counters(rows, E)) * 4, s));
    MOE_CUDA(launch_ffn_decode(x_perm, nullptr, rows, offsets, fc1_q, fc2_q, rows, H, E, I, act_buf,
                               y_perm, ctr, err, nullptr, nullptr, 0, nullptr, s, ep));
    return MOE_OK;
}

moe_status convert_chunked_to_interleaved(const void* src, void* dst, int E, int I, int H,
                                          moe_dtype dt, void* stream) {
    if (E <= 0 || I <= 0 || H <= 0 || H % 8 || !valid_dtype(dt)) return MOE_ERR_INVALID_ARG;
    if (!src || !dst || !aligned(src, 16) || !aligned(dst, 16)) return MOE_ERR_INVALID_ARG;
    const size_t bytes = static_cast<size_t>(E) * 2 * I * H * elem_size(dt);
    const uintptr_t a = reinterpret_cast<uintptr_t>(src), b = reinterpret_cast<uintptr_t>(dst);
    if (a < b + bytes && b < a + bytes) return MOE_ERR_INVALID_ARG;   // overlap
    MOE_CUDA(launch_convert(src, dst, E, I, H, static_cast<int>(elem_size(dt)),
                            static_cast<cudaStream_t>(stream)));
    return MOE_OK;
}

moe_status moe_get_error(const int32_t* err_word, void* stream, int32_t* bits) {
    if (!err_word) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t v = 0;
    if (cudaMemcpyAsync(&v, err_word, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
    if (bits) *bits = v;
    if (v & MOE_DEVERR_TIMEOUT) return MOE_ERR_TIMEOUT;
    if (v) return MOE_ERR_DEVICE;
    return MOE_OK;
}

}  // extern "C"
