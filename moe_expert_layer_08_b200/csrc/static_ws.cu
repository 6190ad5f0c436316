// static_ws.cu -- moe_forward_static: the MoE layer for callers that cannot
// allocate device memory.
//
// Who cannot allocate: code that runs while a CUDA graph is being captured
// (cudaMalloc is not a stream operation and is not allowed there), serving
// runtimes that reserve all device memory for their own pools at start-up and
// forbid any later allocation on the request path, and plug-ins called from
// inside another framework's operator that have no access to that framework's
// allocator and must not call cudaMalloc, which can synchronise the device.
// Such a caller still owns its inputs and outputs; only the layer's scratch
// (routing metadata, gathered activations, the SwiGLU output and the GEMM2
// rows) comes from here: one file-scope device array of
// MOE_STATIC_WORKSPACE_BYTES, which every GPU that loads the library holds
// until the process exits.
#include <mutex>

#include "moe.h"
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

// The scratch itself.  In host code this name is only a host-side stand-in
// for the device array, never a device address: the device address comes from
// cudaGetSymbolAddress below, once per device.
__device__ __align__(256) uint8_t g_static_workspace[MOE_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
uint8_t *g_static_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch on the current device (looked up on the first
// call per device, with that device current).
moe_status_t static_workspace_of_current_device(uint8_t **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> g(g_mu);
    if (!g_static_ptr[dev]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_static_workspace);
        if (e != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
        g_static_ptr[dev] = static_cast<uint8_t *>(p);
    }
    *out = g_static_ptr[dev];
    return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status_t moe_forward_static(const void *x_fp8, const void *x_sf, const int64_t *topk_idx,
                                           const float *topk_w, const void *l1_t, const void *l2_t,
                                           void *out_bf16, int T, int E, int k, int H, int I,
                                           int32_t *expert_stats, void *const *stage_events,
                                           moe_stream_t stream) {
    moe_status_t s = check_shape(E, H, I);
    if (s != MOE_OK) return s;
    if (T < 0 || k <= 0 || k > E) return MOE_ERR_INVALID_ARG;
    if (int64_t(T) * k > int64_t(0x7FFFFFFF) / 2) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (T == 0) return MOE_OK;
    if (!x_fp8 || !x_sf || !topk_idx || !topk_w || !l1_t || !l2_t || !out_bf16) return MOE_ERR_INVALID_ARG;
    if (!aligned(x_fp8, 16) || !aligned(x_sf, 4) || !aligned(topk_idx, 8) || !aligned(topk_w, 4) ||
        !aligned(l1_t, 256) || !aligned(l2_t, 256) || !aligned(out_bf16, 16) ||
        (expert_stats && !aligned(expert_stats, 4)))
        return MOE_ERR_INVALID_ARG;
    // Sizes beyond the fixed scratch are rejected before any device work.
    if (ws_layout(T, E, k, H, I).total > size_t(MOE_STATIC_WORKSPACE_BYTES)) return MOE_ERR_WORKSPACE_TOO_SMALL;
    s = use_device_of(out_bf16);
    if (s != MOE_OK) return s;
    uint8_t *ws = nullptr;
    s = static_workspace_of_current_device(&ws);
    if (s != MOE_OK) return s;
    // Nothing in the scratch has to start at zero: every region the layer
    // reads is written earlier in the same call (routing header included).
    const moe_activation_t swiglu = {MOE_ACT_SWIGLU, 1.0f, 0.0f};
    const moe_weights_t w = {MOE_LAYOUT_PACKETS, l1_t, nullptr, l2_t, nullptr};
    return run_layer(x_fp8, x_sf, topk_idx, topk_w, w, out_bf16, T, E, k, H, I, ws, expert_stats, stage_events,
                     stream, swiglu, false);
}

extern "C" moe_status_t moe_check_device_error_static(int device, moe_stream_t stream) {
    if (device < 0 || device >= kMaxDevices) return MOE_ERR_INVALID_ARG;
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) return MOE_ERR_CUDA;
    if (cur != device && cudaSetDevice(device) != cudaSuccess) return MOE_ERR_CUDA;
    uint8_t *ws = nullptr;
    const moe_status_t s = static_workspace_of_current_device(&ws);
    if (s != MOE_OK) return s;
    // The error word is the first word of the scratch's header, as in a caller workspace.
    return moe_check_device_error(ws, stream);
}
