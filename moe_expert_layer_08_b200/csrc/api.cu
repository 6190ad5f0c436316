// api.cu -- the C ABI declared in include/moe.h: host validation (fails closed
// before any CUDA call, as the DeepGEMM PR #394 "Scope and fallback" section
// asks of unsupported shapes), workspace layout, TMA descriptor encoding and
// the launch sequence of one layer.
#include <cmath>
#include <mutex>
#include <vector>

#include "moe.h"
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

WsLayout ws_layout(int T, int E, int k, int H, int I) {
    WsLayout L;
    L.R = int64_t(T) * k;
    L.nb = int((L.R + kRouteBlock - 1) / kRouteBlock);
    if (L.nb < 1) L.nb = 1;
    // Small per-expert loads (decode) use 32-row chunks and the kN = 32 GEMMs,
    // large ones 160-row chunks (plus the side list).  The chunk-count bound is
    // taken for 32-row chunks either way; the scale regions are sized for the
    // chunking in use, which still grows monotonically with T (at the switch
    // the 160-row bound, (R/160 + E) x 1 KB per K block, exceeds the 32-row one,
    // (R/32 + E) x 512 B with R = 8E).
    L.chunk_rows = L.R <= int64_t(8) * E ? kChunkRowsSmall : kChunkRows;
    L.max_chunks = (L.R + kChunkRowsSmall - 1) / kChunkRowsSmall + (L.R < E ? L.R : E);
    const size_t R = size_t(L.R > 0 ? L.R : 1);
    const size_t MC = size_t(L.max_chunks > 0 ? L.max_chunks : 1);
    size_t o = kHdrBytes;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o += align_up(bytes, 256);
        return at;
    };
    L.off_count = take(sizeof(int) * size_t(E));
    L.off_offset = take(sizeof(int) * size_t(E + 1));
    L.off_chunk_base = take(sizeof(int) * size_t(E + 1));
    L.off_chunks = take(sizeof(int4) * MC);
    L.off_hist = take(sizeof(int) * size_t(L.nb) * size_t(E));
    L.off_bad = take(sizeof(int) * size_t(L.nb));
    L.off_lrank = take(sizeof(int) * R);
    L.off_perm = take(sizeof(int) * R);
    L.off_inv = take(sizeof(int) * R);
    L.off_rowinfo = take(sizeof(int4) * R);
    L.Rp = L.R > kChunkRows ? L.R : kChunkRows;  // at least the largest activation box
    L.kbh = H / kTileK > 2 ? H / kTileK : 2;
    L.kbi = I / kTileK > 2 ? I / kTileK : 2;
    L.off_xg = take(size_t(L.Rp) * size_t(L.kbh) * kTileK);
    // scale blocks per K block: (chunk bound) x (image bytes) of the chunking in use
    const size_t sf_small = MC * size_t(act_sf_bytes(kChunkRowsSmall));
    const size_t mc_large = size_t((L.R + kChunkRows - 1) / kChunkRows + (L.R < E ? L.R : E));
    const size_t sf_large = (mc_large > 0 ? mc_large : 1) * size_t(act_sf_bytes(kChunkRows));
    const size_t sf_per_kb = L.chunk_rows == kChunkRowsSmall ? sf_small : sf_large;
    // twice that: NVFP4 operands have four images per 256 K, two per 128
    L.off_xg_sf = take(2 * sf_per_kb * size_t(H / kTileK));
    L.off_hq = take(size_t(L.Rp) * size_t(L.kbi) * kTileK);
    L.off_hq_sf = take(2 * sf_per_kb * size_t(I / kTileK));
    L.off_y = take(R * size_t(H) * 2);
    L.off_part = take(size_t(kMaxSplitUnits) * kPartUnitFloats * sizeof(float));
    // side list (large batches only): one 32-row chunk per lightly loaded expert
    L.side = L.chunk_rows == kChunkRows;
    L.max_side = L.side ? (L.R < E ? L.R : E) : 0;
    const size_t MS = size_t(L.max_side);
    L.off_chunks_s = take(sizeof(int4) * MS);
    L.off_xg_sf_s = take(2 * MS * size_t(act_sf_bytes(kChunkRowsSmall)) * size_t(H / kTileK));
    L.off_hq_sf_s = take(2 * MS * size_t(act_sf_bytes(kChunkRowsSmall)) * size_t(I / kTileK));
    L.total = o;
    return L;
}

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// FP4 weight bodies as a 4D tensor of 4-bit elements (128 K, rows, tile a,
// K block b); a box (128, box_rows, box_a, kblocks) lands in shared memory as
// 128-row slots b * 2 + a, each element expanded to one byte, 128-byte
// swizzle. The GEMMs read every layout through such a box:
//   packets:   (128 K, 128 rows, slot [8704 B], K-tile pair [17408 B]), box (128, 128, 2, kKB)
//   L1 rows:   (128 K, rows E*2I - I [H/2 B], gate/up [I rows], K block [64 B]), box (128, 128, 2, kKB)
//   L2 rows:   (128 K, rows E*H [I/2 B], 1, K block [64 B]), box (128, 256, 1, kKB): two adjacent
//              tiles as one 256-row box, so an odd last tile of the last expert reads zeros
bool encode_weights4(CUtensorMap *m, const void *base, uint64_t rows, uint64_t row_stride, uint64_t a_dim,
                     uint64_t a_stride, uint64_t b_dim, uint64_t b_stride, int box_rows, int box_a, int kblocks) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    const cuuint64_t dims[4] = {cuuint64_t(kTileK), rows, a_dim, b_dim};
    const cuuint64_t strides[3] = {row_stride, a_stride, b_stride};
    const cuuint32_t box[4] = {cuuint32_t(kTileK), cuuint32_t(box_rows), cuuint32_t(box_a), cuuint32_t(kblocks)};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 4, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// NVFP4 packets: bodies as bytes (128 B, 128 rows, slot, K-tile pair), box
// (128, 128, 2, 1) = both tiles of one 256-K block; their scale images as
// words (128, image, packet) from the first image, box (128, 4, 2).
bool encode_nv_packets(CUtensorMap *m, const void *base, int64_t num_packets) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    const cuuint64_t dims[4] = {128, cuuint64_t(kTileRows), 2, cuuint64_t(num_packets / 2)};
    const cuuint64_t strides[3] = {128, cuuint64_t(kNvPacketBytes), cuuint64_t(2 * kNvPacketBytes)};
    const cuuint32_t box[4] = {128, cuuint32_t(kTileRows), 2, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
bool encode_nv_packet_sf(CUtensorMap *m, const void *base, int64_t num_packets) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    const uint8_t *sf0 = static_cast<const uint8_t *>(base) + kNvPacketBody;
    const cuuint64_t dims[3] = {cuuint64_t(kSfBlockBytes / 4), cuuint64_t(kNvImages), cuuint64_t(num_packets)};
    const cuuint64_t strides[2] = {cuuint64_t(kSfBlockBytes), cuuint64_t(kNvPacketBytes)};
    const cuuint32_t box[3] = {cuuint32_t(kSfBlockBytes / 4), cuuint32_t(kNvImages), 2};
    const cuuint32_t estr[3] = {1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint8_t *>(sf0), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Scale blocks as 32-bit words [packet][row_words]: packets (row_words 2176,
// blocks at word 2048) or the row-major layout's separate arrays (row_words
// 128); a box of 128 words moves one 512-byte block, `depth` packets per load.
bool encode_packet_sf(CUtensorMap *m, const void *base, int64_t num_packets, int depth, int row_words) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    const cuuint64_t dims[2] = {cuuint64_t(row_words), cuuint64_t(num_packets)};
    const cuuint64_t strides[1] = {cuuint64_t(row_words) * 4};
    const cuuint32_t box[2] = {cuuint32_t(kPacketSf / 4), cuuint32_t(depth)};
    const cuuint32_t estr[2] = {1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// FP8 activations stored K-block-major, [kblocks][rows][128] bytes, as a 3D
// tensor (128 bytes, rows, K blocks); one box moves `box_rows` rows of
// `depth` consecutive K blocks.
bool encode_act(CUtensorMap *m, const void *base, int64_t rows, int64_t kblocks, int depth, int box_rows) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    const cuuint64_t dims[3] = {cuuint64_t(kTileK), cuuint64_t(rows), cuuint64_t(kblocks)};
    const cuuint64_t strides[2] = {cuuint64_t(kTileK), cuuint64_t(rows) * kTileK};
    const cuuint32_t box[3] = {cuuint32_t(kTileK), cuuint32_t(box_rows), cuuint32_t(depth)};
    const cuuint32_t estr[3] = {1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

}  // namespace

bool encode_bf16_rows(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows, int box_rows) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    const cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
    const cuuint64_t strides[1] = {cuuint64_t(cols * 2)};
    const cuuint32_t box[2] = {64, cuuint32_t(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() {
    static std::mutex mu;
    static int cache[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> g(mu);
    if (dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        cache[dev] = n > 0 ? n : 148;
    }
    return cache[dev];
}

cudaError_t set_max_dynamic_smem(const void *kernel, int bytes) {
    struct Done {
        const void *kernel;
        int dev, bytes;
    };
    static std::mutex mu;
    static std::vector<Done> done;
    int dev = 0;
    const cudaError_t ge = cudaGetDevice(&dev);
    if (ge != cudaSuccess) return ge;
    std::lock_guard<std::mutex> g(mu);
    for (const Done &d : done)
        if (d.kernel == kernel && d.dev == dev && d.bytes >= bytes) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done.push_back({kernel, dev, bytes});
    return e;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

moe_status_t check_shape(int E, int H, int I) {
    if (E <= 0 || H <= 0 || I <= 0) return MOE_ERR_INVALID_ARG;
    if (H % kTileK != 0 || I % kTileK != 0 || I > kMaxI || E > kMaxExperts) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (int64_t(H) * 2 * I > (int64_t(1) << 40)) return MOE_ERR_UNSUPPORTED_SHAPE;
    return MOE_OK;
}

// Make the device that owns `p` current (the library carries its own runtime
// state, so the caller's current device is not visible to it).
moe_status_t use_device_of(const void *p) {
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_INVALID_ARG;
    }
    if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged) return MOE_ERR_INVALID_ARG;
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) return MOE_ERR_CUDA;
    if (cur != attr.device && cudaSetDevice(attr.device) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
}

// The launch sequence of one layer on a validated workspace (shared by the
// entry points that run the layer).  The workspace's device must be current.
moe_status_t run_layer(const void *x_fp8, const void *x_sf, const int64_t *topk_idx, const float *topk_w,
                       const moe_weights_t &w, void *out_bf16, int T, int E, int k, int H, int I,
                       uint8_t *ws, int32_t *expert_stats, void *const *stage_events, moe_stream_t stream,
                       const moe_activation_t &act, bool nvfp4) {
    const WsLayout L = ws_layout(T, E, k, H, I);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    size_t l1_bytes = 0, l2_bytes = 0;
    if (nvfp4)
        moe_transformed_weight_bytes_nvfp4(E, H, I, &l1_bytes, &l2_bytes);
    else
        moe_transformed_weight_bytes(E, H, I, &l1_bytes, &l2_bytes);
    const size_t pkt_bytes = nvfp4 ? kNvPacketBytes : kPacketBytes;
    const int64_t np1 = int64_t(l1_bytes / pkt_bytes), np2 = int64_t(l2_bytes / pkt_bytes);
    const int d1 = gemm_packets_per_stage(true, L.chunk_rows, nvfp4);
    const int d2 = gemm_packets_per_stage(false, L.chunk_rows, nvfp4);
    const int dk = gemm_kblocks_per_stage(L.chunk_rows, nvfp4);
    // operand rows are stored in 128-byte column blocks (128 FP8 or 256 FP4 elements)
    const int64_t kbh = nvfp4 ? H / kNvTileK : L.kbh, kbi = nvfp4 ? I / kNvTileK : L.kbi;
    CUtensorMap tm_w1, tm_w2, tm_s1, tm_s2, tm_xg, tm_hq, tm_xg_full, tm_hq_full;
    const bool rowmajor = w.layout == MOE_LAYOUT_ROW_MAJOR;
    // weight maps whose boxes move b1 / b2 packets (a stage of that GEMM variant)
    auto encode_w = [&](int b1, int b2, CUtensorMap *w1, CUtensorMap *w2, CUtensorMap *s1, CUtensorMap *s2) {
        if (nvfp4)
            return encode_nv_packets(w1, w.l1, np1) && encode_nv_packets(w2, w.l2, np2) &&
                   encode_nv_packet_sf(s1, w.l1, np1) && encode_nv_packet_sf(s2, w.l2, np2);
        if (rowmajor) {
            const uint64_t e = uint64_t(E), h = uint64_t(H), i = uint64_t(I);
            return encode_weights4(w1, w.l1, e * 2 * i - i, h / 2, 2, i * h / 2, h / kTileK, kTileK / 2, kTileRows, 2,
                                   b1 / 2) &&
                   encode_weights4(w2, w.l2, e * h, i / 2, 1, e * h * i / 2, i / kTileK, kTileK / 2, 2 * kTileRows, 1,
                                   b2 / 2) &&
                   encode_packet_sf(s1, w.l1_sf, np1, b1, kPacketSf / 4) &&
                   encode_packet_sf(s2, w.l2_sf, np2, b2, kPacketSf / 4);
        }
        return encode_weights4(w1, w.l1, kTileRows, kTileK / 2, 2, kPacketBytes, uint64_t(np1 / 2), 2 * kPacketBytes,
                               kTileRows, 2, b1 / 2) &&
               encode_weights4(w2, w.l2, kTileRows, kTileK / 2, 2, kPacketBytes, uint64_t(np2 / 2), 2 * kPacketBytes,
                               kTileRows, 2, b2 / 2) &&
               encode_packet_sf(s1, w.l1, np1, b1, kPacketBytes / 4) &&
               encode_packet_sf(s2, w.l2, np2, b2, kPacketBytes / 4);
    };
    bool ok = encode_w(d1, d2, &tm_w1, &tm_w2, &tm_s1, &tm_s2);
    if (!ok ||
        !encode_act(&tm_xg, ws + L.off_xg, L.Rp, kbh, dk, kActBoxRows) ||
        !encode_act(&tm_hq, ws + L.off_hq, L.Rp, kbi, dk, kActBoxRows) ||
        !encode_act(&tm_xg_full, ws + L.off_xg, L.Rp, kbh, dk, L.chunk_rows) ||
        !encode_act(&tm_hq_full, ws + L.off_hq, L.Rp, kbi, dk, L.chunk_rows))
        return MOE_ERR_CUDA;
    // the side list's 32-row kernels: their own box depths
    CUtensorMap tm_w1s, tm_w2s, tm_s1s, tm_s2s, tm_xgs, tm_hqs;
    if (L.side) {
        const int dks = gemm_kblocks_per_stage(kChunkRowsSmall, nvfp4);
        if (!encode_w(gemm_packets_per_stage(true, kChunkRowsSmall, nvfp4),
                      gemm_packets_per_stage(false, kChunkRowsSmall, nvfp4), &tm_w1s, &tm_w2s, &tm_s1s, &tm_s2s) ||
            !encode_act(&tm_xgs, ws + L.off_xg, L.Rp, kbh, dks, kActBoxRows) ||
            !encode_act(&tm_hqs, ws + L.off_hq, L.Rp, kbi, dks, kActBoxRows))
            return MOE_ERR_CUDA;
    }

    auto record = [&](int i) -> cudaError_t {
        if (!stage_events || !stage_events[i]) return cudaSuccess;
        return cudaEventRecord(static_cast<cudaEvent_t>(stage_events[i]), st);
    };
    const int sms = num_sms();
    const int64_t items1 = L.max_chunks * (I / kTileRows);
    const int64_t items2 = L.max_chunks * (H / kTileRows);
    const int grid1 = int(items1 < sms ? items1 : sms);
    const int grid2 = int(items2 < sms ? items2 : sms);
    const int64_t items1s = L.max_side * (I / kTileRows), items2s = L.max_side * ((H / kTileRows + 1) / 2);
    const int grid1s = int(items1s < sms ? items1s : sms), grid2s = int(items2s < sms ? items2s : sms);

    cudaError_t e = record(0);
    if (e == cudaSuccess)
        e = launch_route(topk_idx, static_cast<const uint8_t *>(x_fp8), static_cast<const uint8_t *>(x_sf), T, k, E,
                         H, ws, L, expert_stats, nvfp4, st);
    if (e == cudaSuccess) e = record(1);
    if (e == cudaSuccess)
        e = launch_gemm(true, tm_w1, tm_s1, tm_xg, tm_xg_full, rowmajor, ws, L, H, I, grid1, st, act, nvfp4);
    if (e == cudaSuccess && L.side)
        e = launch_gemm(true, tm_w1s, tm_s1s, tm_xgs, tm_xgs, rowmajor, ws, L, H, I, grid1s > 0 ? grid1s : 1, st, act,
                        nvfp4, true);
    if (e == cudaSuccess) e = record(2);
    if (e == cudaSuccess)
        e = launch_gemm(false, tm_w2, tm_s2, tm_hq, tm_hq_full, rowmajor, ws, L, H, I, grid2, st, act, nvfp4);
    if (e == cudaSuccess && L.side)
        e = launch_gemm(false, tm_w2s, tm_s2s, tm_hqs, tm_hqs, rowmajor, ws, L, H, I, grid2s > 0 ? grid2s : 1, st, act,
                        nvfp4, true);
    if (e == cudaSuccess) e = record(3);
    if (e == cudaSuccess) e = launch_combine(ws, L, topk_w, T, k, H, out_bf16, st);
    if (e == cudaSuccess) e = record(4);
    return cuda_status(e);
}

}  // namespace moe

using namespace moe;

extern "C" {

const char *moe_status_string(int status) {
    switch (status) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
        case MOE_ERR_UNSUPPORTED_SHAPE: return "MOE_ERR_UNSUPPORTED_SHAPE";
        case MOE_ERR_WORKSPACE_TOO_SMALL: return "MOE_ERR_WORKSPACE_TOO_SMALL";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
        case MOE_ERR_BAD_ROUTING: return "MOE_ERR_BAD_ROUTING";
        case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT";
        default: return "MOE_ERR_UNKNOWN";
    }
}

int moe_abi_version(void) { return 1; }

moe_status_t moe_quantize_fp8(const void *x, int64_t rows, int64_t cols, void *q, void *sf, moe_stream_t stream) {
    if (rows < 0 || cols < 0) return MOE_ERR_INVALID_ARG;
    if (cols % 32 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (rows == 0 || cols == 0) return MOE_OK;
    if (!x || !q || !sf || !aligned(x, 16) || !aligned(q, 16)) return MOE_ERR_INVALID_ARG;
    moe_status_t s = use_device_of(q);
    if (s != MOE_OK) return s;
    return cuda_status(launch_quantize(x, rows, cols, q, sf, true, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_quantize_fp4(const void *w, int64_t rows, int64_t cols, void *q, void *sf, moe_stream_t stream) {
    if (rows < 0 || cols < 0) return MOE_ERR_INVALID_ARG;
    if (cols % 32 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (rows == 0 || cols == 0) return MOE_OK;
    if (!w || !q || !sf || !aligned(w, 16) || !aligned(q, 16)) return MOE_ERR_INVALID_ARG;
    moe_status_t s = use_device_of(q);
    if (s != MOE_OK) return s;
    return cuda_status(launch_quantize(w, rows, cols, q, sf, false, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_transformed_weight_bytes(int E, int H, int I, size_t *l1_bytes, size_t *l2_bytes) {
    const moe_status_t s = check_shape(E, H, I);
    if (s != MOE_OK) return s;
    // L1: (I/128 gate/up tile pairs) x (H/128 K tiles) x 2 packets per expert;
    // L2: (H/128 tiles rounded up to pairs) x (I/128 K tiles) packets per expert
    const size_t l1_packets = size_t(I / kTileRows) * size_t(H / kTileK) * 2;
    const size_t l2_packets = size_t((H / kTileRows + 1) / 2) * size_t(I / kTileK) * 2;
    if (l1_bytes) *l1_bytes = size_t(E) * l1_packets * kPacketBytes;
    if (l2_bytes) *l2_bytes = size_t(E) * l2_packets * kPacketBytes;
    return MOE_OK;
}

moe_status_t moe_transform_weights(const void *l1, const void *l1_sf, const void *l2, const void *l2_sf, int E,
                                   int H, int I, void *l1_t, void *l2_t, moe_stream_t stream) {
    const moe_status_t s = check_shape(E, H, I);
    if (s != MOE_OK) return s;
    if (!l1 || !l1_sf || !l2 || !l2_sf || !l1_t || !l2_t) return MOE_ERR_INVALID_ARG;
    if (!aligned(l1, 16) || !aligned(l2, 16) || !aligned(l1_sf, 4) || !aligned(l2_sf, 4) || !aligned(l1_t, 256) ||
        !aligned(l2_t, 256))
        return MOE_ERR_INVALID_ARG;
    const moe_status_t d = use_device_of(l1_t);
    if (d != MOE_OK) return d;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = launch_transform(l1, l1_sf, E, 2 * I, H, I / kTileRows, false, I, l1_t, true, st);
    if (e == cudaSuccess) e = launch_transform(l2, l2_sf, E, H, I, (H / kTileRows + 1) / 2, true, 0, l2_t, true, st);
    return cuda_status(e);
}

moe_status_t moe_transformed_scale_bytes(int E, int H, int I, size_t *l1_sf_bytes, size_t *l2_sf_bytes) {
    size_t a = 0, b = 0;
    const moe_status_t s = moe_transformed_weight_bytes(E, H, I, &a, &b);
    if (s != MOE_OK) return s;
    if (l1_sf_bytes) *l1_sf_bytes = a / kPacketBytes * kPacketSf;
    if (l2_sf_bytes) *l2_sf_bytes = b / kPacketBytes * kPacketSf;
    return MOE_OK;
}

moe_status_t moe_transform_scales(const void *l1_sf, const void *l2_sf, int E, int H, int I, void *l1_sf_t,
                                  void *l2_sf_t, moe_stream_t stream) {
    const moe_status_t s = check_shape(E, H, I);
    if (s != MOE_OK) return s;
    if (!l1_sf || !l2_sf || !l1_sf_t || !l2_sf_t) return MOE_ERR_INVALID_ARG;
    if (!aligned(l1_sf, 4) || !aligned(l2_sf, 4) || !aligned(l1_sf_t, 256) || !aligned(l2_sf_t, 256))
        return MOE_ERR_INVALID_ARG;
    const moe_status_t d = use_device_of(l1_sf_t);
    if (d != MOE_OK) return d;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = launch_transform(nullptr, l1_sf, E, 2 * I, H, I / kTileRows, false, I, l1_sf_t, false, st);
    if (e == cudaSuccess)
        e = launch_transform(nullptr, l2_sf, E, H, I, (H / kTileRows + 1) / 2, true, 0, l2_sf_t, false, st);
    return cuda_status(e);
}

moe_status_t moe_workspace_bytes(int T_max, int E, int k, int H, int I, size_t *bytes) {
    const moe_status_t s = check_shape(E, H, I);
    if (s != MOE_OK) return s;
    if (T_max < 0 || k <= 0 || k > E || !bytes) return MOE_ERR_INVALID_ARG;
    if (int64_t(T_max) * k > int64_t(0x7FFFFFFF) / 2) return MOE_ERR_UNSUPPORTED_SHAPE;
    *bytes = ws_layout(T_max, E, k, H, I).total;
    return MOE_OK;
}

moe_status_t moe_forward_kernel_launches(int T, int E, int k, int H, int I, int *launches) {
    const moe_status_t s = check_shape(E, H, I);
    if (s != MOE_OK) return s;
    if (T < 0 || k <= 0 || k > E || !launches) return MOE_ERR_INVALID_ARG;
    if (int64_t(T) * k > int64_t(0x7FFFFFFF) / 2) return MOE_ERR_UNSUPPORTED_SHAPE;
    // route + gather, GEMM1, GEMM2 (each twice with a side list: T*k > 8E), combine
    const bool side = int64_t(T) * k > int64_t(8) * E;
    *launches = T == 0 ? 0 : route_kernel_launches(T * k) + (side ? 5 : 3);
    return MOE_OK;
}

moe_status_t moe_forward(const void *x_fp8, const void *x_sf, const int64_t *topk_idx, const float *topk_w,
                         const void *l1_t, const void *l2_t, void *out_bf16, int T, int E, int k, int H, int I,
                         void *workspace, size_t ws_bytes, int32_t *expert_stats, void *const *stage_events,
                         moe_stream_t stream) {
    return moe_forward_act(x_fp8, x_sf, topk_idx, topk_w, l1_t, l2_t, out_bf16, T, E, k, H, I, workspace, ws_bytes,
                           expert_stats, stage_events, nullptr, stream);
}

moe_status_t moe_forward_act(const void *x_fp8, const void *x_sf, const int64_t *topk_idx, const float *topk_w,
                             const void *l1_t, const void *l2_t, void *out_bf16, int T, int E, int k, int H, int I,
                             void *workspace, size_t ws_bytes, int32_t *expert_stats, void *const *stage_events,
                             const moe_activation_t *activation, moe_stream_t stream) {
    const moe_weights_t w = {MOE_LAYOUT_PACKETS, l1_t, nullptr, l2_t, nullptr};
    return moe_forward_weights(x_fp8, x_sf, topk_idx, topk_w, &w, out_bf16, T, E, k, H, I, workspace, ws_bytes,
                               expert_stats, stage_events, activation, stream);
}

moe_status_t moe_forward_weights(const void *x_fp8, const void *x_sf, const int64_t *topk_idx, const float *topk_w,
                                 const moe_weights_t *weights, void *out_bf16, int T, int E, int k, int H, int I,
                                 void *workspace, size_t ws_bytes, int32_t *expert_stats,
                                 void *const *stage_events, const moe_activation_t *activation,
                                 moe_stream_t stream) {
    if (!weights) return MOE_ERR_INVALID_ARG;
    const moe_weights_t w = *weights;
    if (w.layout == MOE_LAYOUT_PACKETS) {
        if (w.l1_sf || w.l2_sf) return MOE_ERR_INVALID_ARG;
    } else if (w.layout == MOE_LAYOUT_ROW_MAJOR) {
        if (!w.l1_sf || !w.l2_sf || !aligned(w.l1_sf, 256) || !aligned(w.l2_sf, 256)) return MOE_ERR_INVALID_ARG;
    } else {
        return MOE_ERR_INVALID_ARG;
    }
    moe_activation_t act = {MOE_ACT_SWIGLU, 1.0f, 0.0f};
    if (activation) {
        act = *activation;
        if (act.kind == MOE_ACT_SITU) {
            if (!(act.beta > 0.0f) || !isfinite(act.beta) || !(act.linear_beta >= 0.0f) || !isfinite(act.linear_beta))
                return MOE_ERR_INVALID_ARG;
        } else if (act.kind != MOE_ACT_SWIGLU) {
            return MOE_ERR_INVALID_ARG;
        }
    }
    moe_status_t s = check_shape(E, H, I);
    if (s != MOE_OK) return s;
    if (T < 0 || k <= 0 || k > E) return MOE_ERR_INVALID_ARG;
    if (int64_t(T) * k > int64_t(0x7FFFFFFF) / 2) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (T == 0) return MOE_OK;
    if (!x_fp8 || !x_sf || !topk_idx || !topk_w || !w.l1 || !w.l2 || !out_bf16 || !workspace)
        return MOE_ERR_INVALID_ARG;
    if (!aligned(x_fp8, 16) || !aligned(x_sf, 4) || !aligned(topk_idx, 8) || !aligned(topk_w, 4) ||
        !aligned(w.l1, 256) || !aligned(w.l2, 256) || !aligned(out_bf16, 16) || !aligned(workspace, 256) ||
        (expert_stats && !aligned(expert_stats, 4)))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(T, E, k, H, I);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    s = use_device_of(workspace);
    if (s != MOE_OK) return s;
    return run_layer(x_fp8, x_sf, topk_idx, topk_w, w, out_bf16, T, E, k, H, I, static_cast<uint8_t *>(workspace),
                     expert_stats, stage_events, stream, act, false);
}

// ---------------------------------------------------------------- NVFP4 variant
static moe_status_t check_shape_nv(int E, int H, int I) {
    const moe_status_t s = check_shape(E, H, I);
    if (s != MOE_OK) return s;
    return (H % kNvTileK || I % kNvTileK) ? MOE_ERR_UNSUPPORTED_SHAPE : MOE_OK;
}

moe_status_t moe_quantize_nvfp4(const void *x, int64_t rows, int64_t cols, void *q, void *sf, moe_stream_t stream) {
    if (rows < 0 || cols < 0) return MOE_ERR_INVALID_ARG;
    if (cols % 16 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (rows == 0 || cols == 0) return MOE_OK;
    if (!x || !q || !sf || !aligned(x, 16) || !aligned(q, 8)) return MOE_ERR_INVALID_ARG;
    moe_status_t s = use_device_of(q);
    if (s != MOE_OK) return s;
    return cuda_status(launch_quantize_nvfp4(x, rows, cols, q, sf, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_transformed_weight_bytes_nvfp4(int E, int H, int I, size_t *l1_bytes, size_t *l2_bytes) {
    const moe_status_t s = check_shape_nv(E, H, I);
    if (s != MOE_OK) return s;
    // L1: (I/128 gate/up tile pairs) x (H/256 K tiles) x 2; L2: (H/256 tile pairs) x (I/256 K tiles) x 2
    if (l1_bytes) *l1_bytes = size_t(E) * size_t(I / kTileRows) * size_t(H / kNvTileK) * 2 * kNvPacketBytes;
    if (l2_bytes) *l2_bytes = size_t(E) * size_t(H / (2 * kTileRows)) * size_t(I / kNvTileK) * 2 * kNvPacketBytes;
    return MOE_OK;
}

moe_status_t moe_transform_weights_nvfp4(const void *l1, const void *l1_sf, const void *l2, const void *l2_sf,
                                         int E, int H, int I, void *l1_t, void *l2_t, moe_stream_t stream) {
    const moe_status_t s = check_shape_nv(E, H, I);
    if (s != MOE_OK) return s;
    if (!l1 || !l1_sf || !l2 || !l2_sf || !l1_t || !l2_t) return MOE_ERR_INVALID_ARG;
    if (!aligned(l1, 16) || !aligned(l2, 16) || !aligned(l1_sf, 4) || !aligned(l2_sf, 4) || !aligned(l1_t, 256) ||
        !aligned(l2_t, 256))
        return MOE_ERR_INVALID_ARG;
    const moe_status_t d = use_device_of(l1_t);
    if (d != MOE_OK) return d;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = launch_transform_nv(l1, l1_sf, E, 2 * I, H, I / kTileRows, false, I, l1_t, st);
    if (e == cudaSuccess) e = launch_transform_nv(l2, l2_sf, E, H, I, H / (2 * kTileRows), true, 0, l2_t, st);
    return cuda_status(e);
}

moe_status_t moe_forward_nvfp4(const void *x_fp4, const void *x_sf, const int64_t *topk_idx, const float *topk_w,
                               const void *l1_t, const void *l2_t, void *out_bf16, int T, int E, int k, int H, int I,
                               void *workspace, size_t ws_bytes, int32_t *expert_stats, void *const *stage_events,
                               const moe_activation_t *activation, moe_stream_t stream) {
    moe_activation_t act = {MOE_ACT_SWIGLU, 1.0f, 0.0f};
    if (activation) {
        act = *activation;
        if (act.kind == MOE_ACT_SITU) {
            if (!(act.beta > 0.0f) || !isfinite(act.beta) || !(act.linear_beta >= 0.0f) || !isfinite(act.linear_beta))
                return MOE_ERR_INVALID_ARG;
        } else if (act.kind != MOE_ACT_SWIGLU) {
            return MOE_ERR_INVALID_ARG;
        }
    }
    moe_status_t s = check_shape_nv(E, H, I);
    if (s != MOE_OK) return s;
    if (T < 0 || k <= 0 || k > E) return MOE_ERR_INVALID_ARG;
    if (int64_t(T) * k > int64_t(0x7FFFFFFF) / 2) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (T == 0) return MOE_OK;
    if (!x_fp4 || !x_sf || !topk_idx || !topk_w || !l1_t || !l2_t || !out_bf16 || !workspace)
        return MOE_ERR_INVALID_ARG;
    if (!aligned(x_fp4, 16) || !aligned(x_sf, 4) || !aligned(topk_idx, 8) || !aligned(topk_w, 4) ||
        !aligned(l1_t, 256) || !aligned(l2_t, 256) || !aligned(out_bf16, 16) || !aligned(workspace, 256) ||
        (expert_stats && !aligned(expert_stats, 4)))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(T, E, k, H, I);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    s = use_device_of(workspace);
    if (s != MOE_OK) return s;
    const moe_weights_t w = {MOE_LAYOUT_PACKETS, l1_t, nullptr, l2_t, nullptr};
    return run_layer(x_fp4, x_sf, topk_idx, topk_w, w, out_bf16, T, E, k, H, I, static_cast<uint8_t *>(workspace),
                     expert_stats, stage_events, stream, act, true);
}

moe_status_t moe_read_routing(const void *workspace, int T, int E, int k, int H, int I, int32_t *count,
                              int32_t *offset, int32_t *perm, int32_t *inv, moe_stream_t stream) {
    moe_status_t s = check_shape(E, H, I);
    if (s != MOE_OK) return s;
    if (!workspace || T < 0 || k <= 0) return MOE_ERR_INVALID_ARG;
    s = use_device_of(workspace);
    if (s != MOE_OK) return s;
    const WsLayout L = ws_layout(T, E, k, H, I);
    const uint8_t *ws = static_cast<const uint8_t *>(workspace);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    if (count) e = cudaMemcpyAsync(count, ws + L.off_count, sizeof(int32_t) * E, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess && offset)
        e = cudaMemcpyAsync(offset, ws + L.off_offset, sizeof(int32_t) * (E + 1), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess && perm && L.R > 0)
        e = cudaMemcpyAsync(perm, ws + L.off_perm, sizeof(int32_t) * L.R, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess && inv && L.R > 0)
        e = cudaMemcpyAsync(inv, ws + L.off_inv, sizeof(int32_t) * L.R, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    return cuda_status(e);
}

// ---------------------------------------------------------------- bounded-wait probe
// One thread waits on a barrier that nothing completes, through the same
// bounded wait every kernel of the library uses, with a short limit: the wait
// gives up, records the timeout in the workspace error word (and `where`) and
// the kernel returns.
__global__ void wait_probe_kernel(int *hdr, unsigned long long timeout_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
    mbar_wait(&bar, 0, &abort_flag, hdr, kProbeWhere, timeout_ns);
}

moe_status_t moe_probe_wait_timeout(void *workspace, size_t ws_bytes, unsigned timeout_us, moe_stream_t stream) {
    if (!workspace || !aligned(workspace, 256) || timeout_us == 0 || timeout_us > 1000000u)
        return MOE_ERR_INVALID_ARG;
    if (ws_bytes < size_t(kHdrBytes)) return MOE_ERR_WORKSPACE_TOO_SMALL;
    moe_status_t s = use_device_of(workspace);
    if (s != MOE_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(workspace, 0, kHdrBytes, st);
    if (e == cudaSuccess) {
        wait_probe_kernel<<<1, 32, 0, st>>>(static_cast<int *>(workspace), 1000ull * timeout_us);
        e = cudaGetLastError();
    }
    return cuda_status(e);
}

// ---------------------------------------------------------------- BF16 shared expert
// header (error word, split counters), h [T][SI] bf16, K-split partial sums
static size_t shared_h_bytes(int T, int SI) { return align_up(size_t(T) * size_t(SI) * 2, 256); }
static size_t shared_ws_bytes(int T, int SI) { return kHdrBytes + shared_h_bytes(T, SI) + shared_part_bytes(T); }

moe_status_t moe_shared_workspace_bytes(int T_max, int SH, int SI, size_t *bytes) {
    if (!bytes || T_max < 0 || SH <= 0 || SI <= 0) return MOE_ERR_INVALID_ARG;
    if (SH % kTileRows || SI % kTileRows) return MOE_ERR_UNSUPPORTED_SHAPE;
    *bytes = shared_ws_bytes(T_max, SI);
    return MOE_OK;
}

moe_status_t moe_shared_forward(const void *x_bf16, const void *l1_bf16, const void *l2_bf16, void *out_bf16, int T,
                                int SH, int SI, const moe_activation_t *activation, void *workspace,
                                size_t ws_bytes, moe_stream_t stream) {
    moe_activation_t act = {MOE_ACT_SWIGLU, 1.0f, 0.0f};
    if (activation) {
        act = *activation;
        if (act.kind == MOE_ACT_SITU) {
            if (!(act.beta > 0.0f) || !isfinite(act.beta) || !(act.linear_beta >= 0.0f) || !isfinite(act.linear_beta))
                return MOE_ERR_INVALID_ARG;
        } else if (act.kind != MOE_ACT_SWIGLU) {
            return MOE_ERR_INVALID_ARG;
        }
    }
    if (T < 0 || SH <= 0 || SI <= 0) return MOE_ERR_INVALID_ARG;
    if (SH % kTileRows || SI % kTileRows) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (T == 0) return MOE_OK;
    if (!x_bf16 || !l1_bf16 || !l2_bf16 || !out_bf16 || !workspace) return MOE_ERR_INVALID_ARG;
    if (!aligned(x_bf16, 16) || !aligned(l1_bf16, 16) || !aligned(l2_bf16, 16) || !aligned(out_bf16, 16) ||
        !aligned(workspace, 256))
        return MOE_ERR_INVALID_ARG;
    if (ws_bytes < shared_ws_bytes(T, SI)) return MOE_ERR_WORKSPACE_TOO_SMALL;
    moe_status_t s = use_device_of(workspace);
    if (s != MOE_OK) return s;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    void *h = ws + kHdrBytes;
    const int kn = shared_block_rows(T);
    CUtensorMap tm_l1, tm_x, tm_l2, tm_h;
    if (!encode_bf16_rows(&tm_l1, l1_bf16, uint64_t(SH), uint64_t(2) * SI, kTileRows) ||
        !encode_bf16_rows(&tm_x, x_bf16, uint64_t(SH), uint64_t(T), kn) ||
        !encode_bf16_rows(&tm_l2, l2_bf16, uint64_t(SI), uint64_t(SH), kTileRows) ||
        !encode_bf16_rows(&tm_h, h, uint64_t(SI), uint64_t(T), kn))
        return MOE_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int *hdr = reinterpret_cast<int *>(ws);
    // no memset: GEMM1 clears the error word, each GEMM the other's split
    // counters (the workspace is zero-filled before its first use)
    float *part = reinterpret_cast<float *>(ws + kHdrBytes + shared_h_bytes(T, SI));
    cudaError_t e = launch_shared(true, tm_l1, tm_x, T, SH, SI, h, hdr, part, act, st);
    if (e == cudaSuccess) e = launch_shared(false, tm_l2, tm_h, T, SH, SI, out_bf16, hdr, part, act, st);
    return cuda_status(e);
}

moe_status_t moe_check_device_error(const void *workspace, moe_stream_t stream) {
    if (!workspace) return MOE_ERR_INVALID_ARG;
    moe_status_t s = use_device_of(workspace);
    if (s != MOE_OK) return s;
    int word = 0;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    if (word & kDevErrTimeout) return MOE_ERR_DEVICE_TIMEOUT;
    if (word & kDevErrBadRouting) return MOE_ERR_BAD_ROUTING;
    return MOE_OK;
}

}  // extern "C"
