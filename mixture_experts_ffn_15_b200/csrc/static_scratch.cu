// moe_forward_static: the whole layer with its scratch in a fixed device array.
//
// Some callers cannot allocate device memory when they run the layer: an engine
// plugin or a serving loop that forbids allocation once it has started (an
// allocation can stall, fragment a pool it does not own, or fail at the worst
// moment), or a plain C host with no allocator of its own that wants to pass
// only its inputs and outputs.  For them this entry point takes no workspace:
// it runs moe_forward on the array below, which the CUDA runtime places in
// device memory when the library's code is loaded on a GPU and which every GPU
// that loads the library keeps until the process exits.
//
// The array is shared by every call on a device and keeps the previous call's
// contents; moe_forward clears the parts that must start at zero (the error word
// and the completion counter) at the start of each call.  Calls whose work can
// overlap on the GPU (two streams, two host threads) race on the array.
#include <mutex>

#include "moe_b200.h"

namespace {

static __device__ __align__(256) unsigned char g_static_scratch[MOE_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {nullptr};
std::mutex g_setup_mutex;

// The array's device address on the current device.  In host code the name
// g_static_scratch only stands for the symbol, so the address is looked up once
// per device with that device current.
moe_status scratch_address(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr)
            return MOE_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_forward_static(const void* hidden, const void* norm_weight,
                                         float norm_eps, const void* router_w,
                                         const float* router_bias, const void* fc1,
                                         const void* fc2, const void* fc1_bias,
                                         const void* fc2_bias, int T, int H, int E, int k, int I,
                                         int normalize, moe_swiglu act,
                                         moe_fc1_layout fc1_layout, moe_dtype dt, void* out,
                                         void* stream) {
    const size_t need = moe_workspace_size(T, H, E, k, I, dt);
    if (need == 0) return MOE_ERR_INVALID_ARG;                    // invalid sizes
    if (need > static_cast<size_t>(MOE_STATIC_SCRATCH_BYTES)) return MOE_ERR_INVALID_ARG;
    void* scratch = nullptr;
    const moe_status st = scratch_address(&scratch);
    if (st != MOE_OK) return st;
    return moe_forward(hidden, norm_weight, norm_eps, router_w, router_bias, fc1, fc2, fc1_bias,
                       fc2_bias, T, H, E, k, I,
                       normalize, act, fc1_layout, dt, out, scratch, static_cast<size_t>(MOE_STATIC_SCRATCH_BYTES),
                       stream);
}
