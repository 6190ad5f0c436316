// moe_internal.h -- host-side declarations shared by the library's translation
// units: the workspace layout and the kernel launchers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

constexpr int kRouteBlock = 256;  // routed slots per routing block

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Workspace layout of one moe_forward call; a pure function of (T, E, k, H, I).
struct WsLayout {
    int64_t R = 0;          // routed slots T*k
    int64_t max_chunks = 0; // upper bound of (expert, <=128-row) work chunks
    int nb = 0;             // routing blocks
    size_t off_count = 0, off_offset = 0, off_chunk_base = 0, off_chunks = 0;
    size_t off_hist = 0, off_bad = 0, off_lrank = 0, off_perm = 0, off_inv = 0;
    size_t off_xg = 0, off_xg_sf = 0, off_hq = 0, off_hq_sf = 0, off_y = 0;
    size_t total = 0;
};

WsLayout ws_layout(int T, int E, int k, int H, int I);

// Kernel launchers (all asynchronous on `stream`; return cudaGetLastError()).
cudaError_t launch_quantize(const void *x, int64_t rows, int64_t cols, void *q, void *sf, bool fp8,
                            cudaStream_t stream);
cudaError_t launch_transform(const void *w, const void *w_sf, int E, int rows_per_expert, int K, int tiles,
                             int halves, int half_rows, void *out, cudaStream_t stream);
cudaError_t launch_route(const int64_t *topk_idx, const uint8_t *x, const uint8_t *x_sf, int T, int k, int E,
                         int H, uint8_t *ws, const WsLayout &L, int32_t *expert_stats, cudaStream_t stream);
cudaError_t launch_gemm(bool gemm1, const CUtensorMap &tmap_w, const CUtensorMap &tmap_act,
                        const uint8_t *w_packets, uint8_t *ws, const WsLayout &L, int H, int I, int grid,
                        cudaStream_t stream);
cudaError_t launch_combine(const uint8_t *ws, const WsLayout &L, const float *topk_w, int T, int k, int H,
                           void *out, cudaStream_t stream);

// Argument checks shared by the entry points.
bool aligned(const void *p, uintptr_t a);
moe_status_t check_shape(int E, int H, int I);
moe_status_t use_device_of(const void *p);

// The launch sequence of one layer on a validated, large-enough workspace of
// the current device.
moe_status_t run_layer(const void *x_fp8, const void *x_sf, const int64_t *topk_idx, const float *topk_w,
                       const void *l1_t, const void *l2_t, void *out_bf16, int T, int E, int k, int H, int I,
                       uint8_t *ws, int32_t *expert_stats, void *const *stage_events, moe_stream_t stream);

}  // namespace moe
