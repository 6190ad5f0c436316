// moe_internal.h -- host-side declarations shared by the library's translation
// units: the workspace layout and the kernel launchers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

constexpr int kRouteBlock = 256;       // routed slots per routing block (large batches)
constexpr int kRouteSmallMax = 1024;   // batches of at most this many slots route in one block

// Launch `kernel` as a programmatic dependent of the preceding work on `stream`
// (its CTAs may start before that work ends; the kernel orders itself with
// griddepcontrol.wait before touching dependent memory).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Workspace layout of one moe_forward call; a pure function of (T, E, k, H, I).
struct WsLayout {
    int64_t R = 0;          // routed slots T*k
    int64_t max_chunks = 0; // upper bound of (expert, <=128-row) work chunks
    int nb = 0;             // routing blocks
    int chunk_rows = 0;     // routed rows per chunk of the main list (32 or 160)
    // Large batches (chunk_rows = 160) also keep a side list: experts with at
    // most kChunkRowsSmall rows get one 32-row chunk there, which the 32-row
    // kernels process (they stream weights faster than the 160-row ones).
    bool side = false;
    int64_t max_side = 0;   // side-list chunks, at most (one per expert)
    int64_t Rp = 0;         // rows of the K-block-major FP8 operands (R, at least one TMA box)
    int kbh = 0, kbi = 0;   // K blocks of those operands (H/128, I/128, at least 2)
    size_t off_count = 0, off_offset = 0, off_chunk_base = 0, off_chunks = 0;
    size_t off_hist = 0, off_bad = 0, off_lrank = 0, off_perm = 0, off_inv = 0, off_rowinfo = 0;
    size_t off_xg = 0, off_xg_sf = 0, off_hq = 0, off_hq_sf = 0, off_y = 0;
    size_t off_part = 0;    // split-unit partial accumulators of the 32-row GEMMs
    size_t off_chunks_s = 0, off_xg_sf_s = 0, off_hq_sf_s = 0;  // side list and its scale images
    size_t total = 0;
};

WsLayout ws_layout(int T, int E, int k, int H, int I);

// Kernel launchers (all asynchronous on `stream`; return cudaGetLastError()).
cudaError_t launch_quantize(const void *x, int64_t rows, int64_t cols, void *q, void *sf, bool fp8,
                            cudaStream_t stream);
cudaError_t launch_quantize_nvfp4(const void *x, int64_t rows, int64_t cols, void *q, void *sf, cudaStream_t stream);
cudaError_t launch_transform_nv(const void *w, const void *w_sf, int E, int rows_per_expert, int K, int groups,
                                bool pairs, int half_rows, void *out, cudaStream_t stream);
// Tile packets (body + scale block, kPacketBytes each) or, with out_body ==
// nullptr, only the 512-byte scale blocks in the same order (row-major layout).
cudaError_t launch_transform(const void *w, const void *w_sf, int E, int rows_per_expert, int K, int groups,
                             bool pairs, int half_rows, void *out, bool with_body, cudaStream_t stream);
// kernels launch_route enqueues for R = T * k routed rows (one-block routing
// up to kRouteSmallMax rows, then the gather; else four routing kernels and
// the gather)
inline int route_kernel_launches(int64_t R) { return R <= kRouteSmallMax ? 2 : 5; }
cudaError_t launch_route(const int64_t *topk_idx, const uint8_t *x, const uint8_t *x_sf, int T, int k, int E,
                         int H, uint8_t *ws, const WsLayout &L, int32_t *expert_stats, bool nvfp4,
                         cudaStream_t stream);
// GEMM1 / GEMM2 over the main chunk list (side = false: chunks of
// L.chunk_rows rows) or the side list (32-row chunks of lightly loaded
// experts); the tensor maps are those of that chunk size.
cudaError_t launch_gemm(bool gemm1, const CUtensorMap &tmap_w, const CUtensorMap &tmap_wsf,
                        const CUtensorMap &tmap_act, const CUtensorMap &tmap_act_full, bool w_rowmajor,
                        uint8_t *ws, const WsLayout &L, int H, int I, int grid, cudaStream_t stream,
                        const moe_activation_t &act, bool nvfp4, bool side = false);
// Weight packets one pipeline stage of that GEMM variant moves (TMA box depth).
int gemm_packets_per_stage(bool gemm1, int chunk_rows, bool nvfp4);
// K blocks (128 operand bytes each) one pipeline stage moves (the activation box depth).
int gemm_kblocks_per_stage(int chunk_rows, bool nvfp4);
constexpr int kActBoxRows = 32;  // activation rows per TMA box
cudaError_t launch_combine(const uint8_t *ws, const WsLayout &L, const float *topk_w, int T, int k, int H,
                           void *out, cudaStream_t stream);

// BF16 shared expert: tokens per work item (32 up to kSharedTinyT tokens, 64
// up to kSharedSmallT, else 128) and the launch of GEMM1 (tmap_w over L1
// [2SI][SH], tmap_act over x [T][SH], out = h [T][SI]) or GEMM2 (L2 [SH][SI],
// h, out = y [T][SH]); the maps' boxes are 128 / shared_block_rows(T) rows of
// 64 bf16.  part: scratch of shared_part_bytes(T) bytes for K-split partial
// sums.
constexpr int kSharedTinyT = 64;
constexpr int kSharedSmallT = 128;
int shared_block_rows(int T);
size_t shared_part_bytes(int T);
cudaError_t launch_shared(bool gemm1, const CUtensorMap &tmap_w, const CUtensorMap &tmap_act, int T, int SH, int SI,
                          void *out, int *hdr, float *part, const moe_activation_t &act, cudaStream_t stream);
// Tensor map of a row-major bf16 matrix [rows][cols]: boxes of 64 columns
// (128 bytes, 128-byte swizzle) x box_rows rows.
bool encode_bf16_rows(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows, int box_rows);

// Multiprocessors of the current device (cached per device).
int num_sms();
// Opts `kernel` in to `bytes` of dynamic shared memory on the current device,
// once per (kernel, device); safe to call from several host threads.
cudaError_t set_max_dynamic_smem(const void *kernel, int bytes);

// Argument checks shared by the entry points.
bool aligned(const void *p, uintptr_t a);
moe_status_t check_shape(int E, int H, int I);
moe_status_t use_device_of(const void *p);

// The launch sequence of one layer on a validated, large-enough workspace of
// the current device.
moe_status_t run_layer(const void *x_fp8, const void *x_sf, const int64_t *topk_idx, const float *topk_w,
                       const moe_weights_t &w, void *out_bf16, int T, int E, int k, int H, int I,
                       uint8_t *ws, int32_t *expert_stats, void *const *stage_events, moe_stream_t stream,
                       const moe_activation_t &act, bool nvfp4);

}  // namespace moe
