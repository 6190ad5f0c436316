// ep.cu -- the per-rank ends of expert parallelism: the dispatch and combine
// phases of "Mega moe fusion with symmetric memory" (Procedure, step 5,
// phases 1 and 5) with the cross-rank exchange left to the caller (an
// all-to-all-v over NCCL between the two calls and after the expert layer).
//
// Ranks own contiguous expert ranges: rank r holds experts [r*E/R, (r+1)*E/R).
// Dispatch runs the layer's routing (the stable counting sort by expert), so
// the routed rows in permutation order are already grouped by destination
// rank; it copies each routed slot's FP8 row, its UE8M0 scales and its local
// expert id into send buffers in that order and writes the per-rank row
// counts.  The receiving rank runs the expert layer over its E/R experts with
// k = 1 and weight 1 (the layer's output for such a row is its bf16 Y row
// unchanged).  Combine takes the returned rows, still in send order, and
// forms out[t] = bf16(sum_j w[t, j] * Y[inv[t*k + j]]) with the layer's own
// combine kernel through the inverse permutation the dispatch left in the
// workspace.
#include <cstring>

#include "ep_internal.h"
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kPackThreads = 256;

// Workspace of the dispatch: the layer's routing regions only (header,
// counts, offsets, chunk lists, histograms, permutation, inverse, gather
// descriptors), with the side chunk list moved down to where the layer's
// gathered activations would start.
WsLayout ep_layout(int T, int E, int k, int H) {
    WsLayout L = ws_layout(T, E, k, H, kTileK);
    L.off_chunks_s = L.off_xg;
    L.total = L.off_chunks_s + align_up(sizeof(int4) * size_t(L.max_side > 0 ? L.max_side : 1), 256);
    return L;
}

// One warp per routed row (rows in permutation order, nrows = offset[E]):
// send row pos <- token perm[pos] / k (row_vec 16-byte vectors, sf_words
// 4-byte scale words), send_eid[pos] = the slot's expert id modulo e_loc.
// Block 0 also writes send_counts[r] = rows for experts [r*e_loc, (r+1)*e_loc).
__global__ void __launch_bounds__(kPackThreads) ep_pack_kernel(const int *__restrict__ perm,
                                                               const int *__restrict__ offset,
                                                               const int64_t *__restrict__ topk_idx, int E, int k,
                                                               int e_loc, int ranks, int row_vec, int sf_words,
                                                               const uint4 *__restrict__ x,
                                                               const uint32_t *__restrict__ x_sf,
                                                               uint4 *__restrict__ send_x,
                                                               uint32_t *__restrict__ send_sf,
                                                               int64_t *__restrict__ send_eid,
                                                               int64_t *__restrict__ send_counts) {
    pdl_wait();
    pdl_trigger();
    if (blockIdx.x == 0)
        for (int r = threadIdx.x; r < ranks; r += blockDim.x)
            send_counts[r] = int64_t(__ldcg(offset + (r + 1) * e_loc)) - __ldcg(offset + r * e_loc);
    constexpr int kWarps = kPackThreads / 32;
    const int lane = threadIdx.x & 31;
    const int64_t nrows = __ldcg(offset + E);  // dropped slots leave no row
    const int64_t nwarps = int64_t(gridDim.x) * kWarps;
    for (int64_t pos = int64_t(blockIdx.x) * kWarps + (threadIdx.x >> 5); pos < nrows; pos += nwarps) {
        const int s = __ldcg(perm + pos);
        const int64_t t = s / k;
        const uint4 *src = x + t * row_vec;
        uint4 *dst = send_x + pos * row_vec;
        for (int v = lane; v < row_vec; v += 32) dst[v] = __ldg(src + v);
        for (int w = lane; w < sf_words; w += 32) send_sf[pos * sf_words + w] = __ldg(x_sf + t * sf_words + w);
        if (lane == 0) send_eid[pos] = __ldg(topk_idx + s) % e_loc;  // routed: the id is in [0, E)
    }
}

// The dispatch over peer memory: one warp per routed row (permutation order)
// writes the row, its scale words and its local expert id straight into the
// receive buffers of the rank d = e / e_loc that holds its expert, at row
// recv_base[d] + (pos - offset[d * e_loc]).  Block 0 also writes the per-rank
// counts (as ep_pack_kernel does), which the caller has already exchanged
// when it computes recv_base; a NULL peer entry skips that rank's rows.
__global__ void __launch_bounds__(kPackThreads) ep_push_kernel(const int *__restrict__ perm,
                                                               const int *__restrict__ offset,
                                                               const int64_t *__restrict__ topk_idx, int E, int k,
                                                               int e_loc, int row_vec, int sf_words,
                                                               const uint4 *__restrict__ x,
                                                               const uint32_t *__restrict__ x_sf,
                                                               uint4 *const *__restrict__ peer_x,
                                                               uint32_t *const *__restrict__ peer_sf,
                                                               int64_t *const *__restrict__ peer_eid,
                                                               const int64_t *__restrict__ recv_base) {
    pdl_wait();
    pdl_trigger();
    constexpr int kWarps = kPackThreads / 32;
    const int lane = threadIdx.x & 31;
    const int64_t nrows = __ldcg(offset + E);
    const int64_t nwarps = int64_t(gridDim.x) * kWarps;
    for (int64_t pos = int64_t(blockIdx.x) * kWarps + (threadIdx.x >> 5); pos < nrows; pos += nwarps) {
        const int s = __ldcg(perm + pos);
        const int64_t t = s / k;
        const int64_t e = __ldg(topk_idx + s);  // routed: in [0, E)
        const int d = int(e / e_loc);
        uint4 *dx = peer_x[d];
        uint32_t *dsf = peer_sf[d];
        int64_t *deid = peer_eid[d];
        if (!dx || !dsf || !deid) continue;
        const int64_t row = __ldcg(recv_base + d) + (pos - __ldcg(offset + d * e_loc));
        const uint4 *src = x + t * row_vec;
        for (int v = lane; v < row_vec; v += 32) dx[row * row_vec + v] = __ldg(src + v);
        for (int w = lane; w < sf_words; w += 32) dsf[row * sf_words + w] = __ldg(x_sf + t * sf_words + w);
        if (lane == 0) deid[row] = e % e_loc;
    }
}

// Per-rank row counts of a finished routing: counts[r] = rows for experts
// [r*e_loc, (r+1)*e_loc).
__global__ void ep_counts_kernel(const int *__restrict__ offset, int e_loc, int ranks,
                                 int64_t *__restrict__ counts) {
    pdl_wait();
    pdl_trigger();
    for (int r = threadIdx.x; r < ranks; r += blockDim.x)
        counts[r] = int64_t(__ldcg(offset + (r + 1) * e_loc)) - __ldcg(offset + r * e_loc);
}

// The combine over peer memory: out[t] = bf16_rne(sum_{j ascending} w[t, j] *
// Y_j) with Y_j read where the expert layer of the row's rank left it: rank
// d = e / e_loc, row recv_base[d] + (pos - offset[d * e_loc]) of peer_y[d]
// (pos = inv[t*k + j], the row's place in this rank's send order).  Blocks
// stride over (token, 1024-column block) tasks; each thread sums 8 columns
// with the arithmetic of the layer's combine.
constexpr int kPeerThreads = 128;
constexpr int kPeerCols = kPeerThreads * 8;

__global__ void __launch_bounds__(kPeerThreads) ep_combine_peers_kernel(
    const __nv_bfloat16 *const *__restrict__ peer_y, const int64_t *__restrict__ recv_base,
    const int *__restrict__ inv, const int *__restrict__ offset, const int64_t *__restrict__ topk_idx,
    const float *__restrict__ topk_w, int k, int H, int e_loc, int col_blocks, int T, __nv_bfloat16 *__restrict__ out) {
    pdl_wait();
    pdl_trigger();
    for (int64_t task = blockIdx.x; task < int64_t(T) * col_blocks; task += gridDim.x) {
        const int64_t t = task / col_blocks;
        const int col = int(task % col_blocks) * kPeerCols + threadIdx.x * 8;
        if (col >= H) continue;
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
        for (int j = 0; j < k; ++j) {
            const int pos = __ldcg(inv + t * k + j);
            if (pos < 0) continue;  // dropped slot
            const int d = int(__ldg(topk_idx + t * k + j) / e_loc);
            const int64_t row = __ldcg(recv_base + d) + (pos - __ldcg(offset + d * e_loc));
            const __nv_bfloat16 *src = peer_y[d];
            if (!src) continue;  // no buffer given for that rank (its rows contribute nothing)
            const uint4 v = __ldcg(reinterpret_cast<const uint4 *>(src + row * H + col));
            const float wv = __ldg(topk_w + t * k + j);
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                acc[2 * i] += wv * __uint_as_float(u[i] << 16);
                acc[2 * i + 1] += wv * __uint_as_float(u[i] & 0xFFFF0000u);
            }
        }
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
            o[i] = *reinterpret_cast<const uint32_t *>(&b);
        }
        *reinterpret_cast<uint4 *>(out + t * H + col) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

moe_status_t check_ep_args(int T, int E, int k, int H) {
    if (T < 0 || E <= 0 || k <= 0 || k > E || H <= 0) return MOE_ERR_INVALID_ARG;
    if (H % kTileK != 0 || E > kMaxExperts) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (int64_t(T) * k > int64_t(0x7FFFFFFF) / 2) return MOE_ERR_UNSUPPORTED_SHAPE;
    return MOE_OK;
}

// The sizes plus a rank count: 1 <= ranks <= E, E a multiple of ranks.
moe_status_t check_ep_args(int T, int E, int k, int H, int ranks) {
    const moe_status_t s = check_ep_args(T, E, k, H);
    if (s != MOE_OK) return s;
    if (ranks <= 0 || ranks > E) return MOE_ERR_INVALID_ARG;
    return E % ranks == 0 ? MOE_OK : MOE_ERR_UNSUPPORTED_SHAPE;
}

// Blocks of the one-warp-per-row kernels for R routed rows: one warp per row
// up to 8 blocks per SM, the warps striding over the rest.
int row_grid(int64_t R) {
    const int64_t want = (R + kPackThreads / 32 - 1) / (kPackThreads / 32);
    const int64_t cap = int64_t(num_sms()) * 8;
    const int64_t g = want < cap ? want : cap;
    return int(g > 0 ? g : 1);
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

moe_status_t moe_ep_workspace_bytes(int T_max, int E, int k, int H, size_t *bytes) {
    if (!bytes) return MOE_ERR_INVALID_ARG;
    const moe_status_t s = check_ep_args(T_max, E, k, H);
    if (s != MOE_OK) return s;
    *bytes = ep_layout(T_max, E, k, H).total;
    return MOE_OK;
}

moe_status_t moe_ep_dispatch(const void *x_fp8, const void *x_sf, const int64_t *topk_idx, int T, int E, int k,
                             int H, int ranks, void *workspace, size_t ws_bytes, void *send_x, void *send_sf,
                             int64_t *send_eid, int64_t *send_counts, moe_stream_t stream) {
    moe_status_t s = check_ep_args(T, E, k, H, ranks);
    if (s != MOE_OK) return s;
    if (!workspace || !send_counts || !aligned(workspace, 256) || !aligned(send_counts, 8))
        return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!x_fp8 || !x_sf || !topk_idx || !send_x || !send_sf || !send_eid || !aligned(x_fp8, 16) ||
                  !aligned(x_sf, 4) || !aligned(topk_idx, 8) || !aligned(send_x, 16) || !aligned(send_sf, 4) ||
                  !aligned(send_eid, 8)))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = ep_layout(T, E, k, H);
    if (T > 0 && ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    s = use_device_of(workspace);
    if (s != MOE_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (T == 0)
        return cudaMemsetAsync(send_counts, 0, sizeof(int64_t) * size_t(ranks), st) == cudaSuccess ? MOE_OK
                                                                                                     : MOE_ERR_CUDA;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    cudaError_t e = launch_routing(topk_idx, k, E, ws, L, nullptr, st);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    const int grid = row_grid(L.R);
    e = launch_pdl(ep_pack_kernel, dim3(unsigned(grid)), dim3(kPackThreads), 0, st,
                   reinterpret_cast<const int *>(ws + L.off_perm), reinterpret_cast<const int *>(ws + L.off_offset),
                   topk_idx, E, k, E / ranks, ranks, H / 16, H / 128, static_cast<const uint4 *>(x_fp8),
                   static_cast<const uint32_t *>(x_sf), static_cast<uint4 *>(send_x), static_cast<uint32_t *>(send_sf),
                   send_eid, send_counts);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_ep_combine(const void *y_bf16, const float *topk_w, int T, int E, int k, int H,
                            const void *workspace, size_t ws_bytes, void *out_bf16, moe_stream_t stream) {
    moe_status_t s = check_ep_args(T, E, k, H);
    if (s != MOE_OK) return s;
    if (T == 0) return MOE_OK;
    if (!y_bf16 || !topk_w || !workspace || !out_bf16 || !aligned(y_bf16, 16) || !aligned(topk_w, 4) ||
        !aligned(workspace, 256) || !aligned(out_bf16, 16))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = ep_layout(T, E, k, H);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    s = use_device_of(workspace);
    if (s != MOE_OK) return s;
    const uint8_t *ws = static_cast<const uint8_t *>(workspace);
    const cudaError_t e = launch_combine_rows(y_bf16, reinterpret_cast<const int *>(ws + L.off_inv), topk_w, T, k, H,
                                              out_bf16, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_ep_combine_peers(const void *const *peer_y, const int64_t *recv_base, const int64_t *topk_idx,
                                  const float *topk_w, int T, int E, int k, int H, int ranks, const void *workspace,
                                  size_t ws_bytes, void *out_bf16, moe_stream_t stream) {
    moe_status_t s = check_ep_args(T, E, k, H, ranks);
    if (s != MOE_OK) return s;
    if (T == 0) return MOE_OK;
    if (!peer_y || !recv_base || !topk_idx || !topk_w || !workspace || !out_bf16 || !aligned(peer_y, 8) ||
        !aligned(recv_base, 8) || !aligned(topk_idx, 8) || !aligned(topk_w, 4) || !aligned(workspace, 256) ||
        !aligned(out_bf16, 16))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = ep_layout(T, E, k, H);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    s = use_device_of(workspace);
    if (s != MOE_OK) return s;
    const uint8_t *ws = static_cast<const uint8_t *>(workspace);
    const int col_blocks = (H + kPeerCols - 1) / kPeerCols;
    const int64_t tasks = int64_t(T) * col_blocks, cap = int64_t(num_sms()) * 16;
    const int64_t grid = tasks < cap ? tasks : cap;
    const cudaError_t e = launch_pdl(ep_combine_peers_kernel, dim3(unsigned(grid)), dim3(kPeerThreads), 0,
                                     reinterpret_cast<cudaStream_t>(stream),
                                     reinterpret_cast<const __nv_bfloat16 *const *>(peer_y), recv_base,
                                     reinterpret_cast<const int *>(ws + L.off_inv),
                                     reinterpret_cast<const int *>(ws + L.off_offset), topk_idx, topk_w, k, H,
                                     E / ranks, col_blocks, T, static_cast<__nv_bfloat16 *>(out_bf16));
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_ep_route(const int64_t *topk_idx, int T, int E, int k, int H, int ranks, void *workspace,
                          size_t ws_bytes, int64_t *send_counts, moe_stream_t stream) {
    moe_status_t s = check_ep_args(T, E, k, H, ranks);
    if (s != MOE_OK) return s;
    if (!workspace || !send_counts || !aligned(workspace, 256) || !aligned(send_counts, 8) ||
        (T > 0 && (!topk_idx || !aligned(topk_idx, 8))))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = ep_layout(T, E, k, H);
    if (T > 0 && ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    s = use_device_of(workspace);
    if (s != MOE_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (T == 0)
        return cudaMemsetAsync(send_counts, 0, sizeof(int64_t) * size_t(ranks), st) == cudaSuccess ? MOE_OK
                                                                                                     : MOE_ERR_CUDA;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    cudaError_t e = launch_routing(topk_idx, k, E, ws, L, nullptr, st);
    if (e == cudaSuccess)
        e = launch_pdl(ep_counts_kernel, dim3(1), dim3(256), 0, st, reinterpret_cast<const int *>(ws + L.off_offset),
                       E / ranks, ranks, send_counts);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_ep_dispatch_peers(const void *x_fp8, const void *x_sf, const int64_t *topk_idx, int T, int E, int k,
                                   int H, int ranks, const void *workspace, size_t ws_bytes,
                                   void *const *peer_x, void *const *peer_sf, int64_t *const *peer_eid,
                                   const int64_t *recv_base, moe_stream_t stream) {
    moe_status_t s = check_ep_args(T, E, k, H, ranks);
    if (s != MOE_OK) return s;
    if (T == 0) return MOE_OK;
    if (!x_fp8 || !x_sf || !topk_idx || !workspace || !peer_x || !peer_sf || !peer_eid || !recv_base ||
        !aligned(x_fp8, 16) || !aligned(x_sf, 4) || !aligned(topk_idx, 8) || !aligned(workspace, 256) ||
        !aligned(peer_x, 8) || !aligned(peer_sf, 8) || !aligned(peer_eid, 8) || !aligned(recv_base, 8))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = ep_layout(T, E, k, H);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    s = use_device_of(workspace);
    if (s != MOE_OK) return s;
    const uint8_t *ws = static_cast<const uint8_t *>(workspace);
    const int grid = row_grid(L.R);
    const cudaError_t e = launch_pdl(
        ep_push_kernel, dim3(unsigned(grid)), dim3(kPackThreads), 0,
        reinterpret_cast<cudaStream_t>(stream), reinterpret_cast<const int *>(ws + L.off_perm),
        reinterpret_cast<const int *>(ws + L.off_offset), topk_idx, E, k, E / ranks, H / 16, H / 128,
        static_cast<const uint4 *>(x_fp8), static_cast<const uint32_t *>(x_sf),
        reinterpret_cast<uint4 *const *>(peer_x), reinterpret_cast<uint32_t *const *>(peer_sf), peer_eid, recv_base);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// ------------------------------------------------------------------ peer buffers
// Mapping the ranks' receive and output buffers into each other's address
// space with CUDA IPC (for moe_ep_dispatch_peers / moe_ep_combine_peers).  A
// buffer may sit anywhere inside its allocation (framework allocators hand
// out pieces of larger blocks): the handle names the whole allocation and the
// offset locates the buffer in it.

static_assert(sizeof(cudaIpcMemHandle_t) == MOE_IPC_HANDLE_BYTES, "IPC handle size");

moe_status_t moe_ipc_handle(const void *ptr, void *handle, size_t *offset) {
    if (!ptr || !handle || !offset) return MOE_ERR_INVALID_ARG;
    moe_status_t s = use_device_of(ptr);
    if (s != MOE_OK) return s;
    typedef CUresult (*RangeFn)(CUdeviceptr *, size_t *, CUdeviceptr);
    static RangeFn range = []() -> RangeFn {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<RangeFn>(p);
    }();
    if (!range) return MOE_ERR_CUDA;
    CUdeviceptr base = 0;
    size_t bytes = 0;
    if (range(&base, &bytes, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS) return MOE_ERR_CUDA;
    cudaIpcMemHandle_t h;
    if (cudaIpcGetMemHandle(&h, reinterpret_cast<void *>(base)) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    memcpy(handle, &h, sizeof(h));
    *offset = size_t(reinterpret_cast<CUdeviceptr>(ptr) - base);
    return MOE_OK;
}

moe_status_t moe_ipc_open(const void *handle, int device, void **base) {
    if (!handle || !base || device < 0) return MOE_ERR_INVALID_ARG;
    if (cudaSetDevice(device) != cudaSuccess) return MOE_ERR_CUDA;
    cudaIpcMemHandle_t h;
    memcpy(&h, handle, sizeof(h));
    if (cudaIpcOpenMemHandle(base, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

moe_status_t moe_ipc_close(void *base) {
    if (!base) return MOE_ERR_INVALID_ARG;
    if (cudaIpcCloseMemHandle(base) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

}  // extern "C"
