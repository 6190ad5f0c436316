// ep_internal.h -- launchers that the layer (api.cu) and the expert-parallel
// dispatch / combine entry points (ep.cu) share: the routing metadata without
// the gather, and the weighted combine over caller-given rows.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_internal.h"

namespace moe {

// Routing metadata for the L.R = T*k slots of topk_idx into the workspace
// regions of L (per-expert counts, offsets, chunk lists, the stable
// permutation and its inverse, the gather descriptors, the error word);
// no row is copied.
cudaError_t launch_routing(const int64_t *topk_idx, int k, int E, uint8_t *ws, const WsLayout &L,
                           int32_t *expert_stats, cudaStream_t stream);

// out[t, :] = bf16_rne(sum_{j ascending} topk_w[t, j] * y[inv[t*k + j], :]),
// fp32 sum, for T > 0 tokens; y is bf16 [*, H] (16-byte aligned rows), an
// inv entry < 0 marks a dropped slot.
cudaError_t launch_combine_rows(const void *y, const int *inv, const float *topk_w, int T, int k, int H, void *out,
                                cudaStream_t stream);

}  // namespace moe
