// route.cu -- routing (per-expert histogram, exclusive scan, stable
// permutation and its inverse, chunk list) and the local gather that replaces
// the cross-rank dispatch of the "Mega MoE" pipeline ("Mega moe fusion with
// symmetric memory", Procedure step 5, phase 1; the "gather-by-expert" step of
// What / Why).  No host synchronisation anywhere.
//
// Small batches (T*k <= 1024 slots): one block does everything
// (route_small_kernel).  Large batches: route_count (per 256-slot block,
// per-expert counts and each slot's rank among the block's earlier slots of
// its expert), route_colscan (one block per expert: that expert's per-block
// bases and its count), route_meta (one block: offsets, chunk list,
// statistics, error word), route_place (perm, inv, per-row gather
// descriptor).  Then gather_kernel copies the FP8 rows of x into permuted
// order (stored K-block-major, [H/128][R][128]) and the UE8M0 scales into
// per-chunk blocks of 512-byte images laid out as the image tcgen05.cp copies
// into TMEM.
//
// Chunks: an expert's rows are cut into chunks of chunk_rows (32 for small
// batches, 160 for large ones) in the main list.  With 160-row chunks the
// experts with at most 32 rows instead get one 32-row chunk in a side list,
// which the 32-row GEMM kernels process; their per-expert chunk base carries
// kSideChunkBit.
//
// Within an expert, routed rows keep ascending slot order t*k+j (a stable
// counting sort), so the metadata is unique and compared bit-exactly.
#include "ep_internal.h"
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

// Exclusive scan of one int per thread over a block of blockDim.x (<= 1024,
// multiple of 32) threads; every thread must call it.
__device__ __forceinline__ int block_exclusive_scan(int v, int *s_warp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nwarps ? s_warp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, w, o);
            if (lane >= o) w += y;
        }
        s_warp[lane] = w;  // inclusive totals of warps 0..lane
    }
    __syncthreads();
    const int before = warp > 0 ? s_warp[warp - 1] : 0;
    const int r = before + x - v;
    __syncthreads();
    return r;
}

// Whether expert e with c rows goes to the side list (one 32-row chunk;
// only with `side` lists, i.e. 160-row main chunks).
__device__ __forceinline__ bool on_side(bool side, int c) { return side && c <= kChunkRowsSmall; }

// Per expert e (one thread each): count c, offset, chunk base (main-list
// index, or side-list index | kSideChunkBit), chunk list entries, statistics.
// cbase / sbase: the expert's first chunk in the main / side list (exclusive
// scans over experts).  Shared by both routing paths.
__device__ __forceinline__ void write_expert_meta(int e, int E, int c, int off, int cbase, int sbase, bool side,
                                                 int chunk_rows, int *count, int *offset, int *chunk_base,
                                                 int4 *chunks, int4 *chunks_s, int *hdr, int32_t *expert_stats) {
    const bool s = on_side(side, c);
    const int nch = s ? 0 : (c + chunk_rows - 1) / chunk_rows;
    const int nside = (s && c > 0) ? 1 : 0;
    count[e] = c;
    offset[e] = off;
    chunk_base[e] = s ? (kSideChunkBit | sbase) : cbase;
    for (int q = 0; q < nch; ++q)
        chunks[cbase + q] = make_int4(e, off + q * chunk_rows, min(chunk_rows, c - q * chunk_rows), 0);
    if (nside) chunks_s[sbase] = make_int4(e, off, c, 0);
    if (expert_stats) expert_stats[e] += c;
    if (e == E - 1) {
        offset[E] = off + c;
        chunk_base[E] = cbase + nch;
        hdr[kHdrNumChunks] = cbase + nch;
        hdr[kHdrNumChunksSide] = sbase + nside;
    }
}

// Gather descriptor of a routed row: token, chunk (in its list), row within
// the chunk, list (0 main, 1 side).
__device__ __forceinline__ int4 row_info(int token, int cb, int local, int chunk_rows) {
    return (cb & kSideChunkBit) ? make_int4(token, cb & ~kSideChunkBit, local, 1)
                                : make_int4(token, cb + local / chunk_rows, local % chunk_rows, 0);
}

// ------------------------------------------------------------------ small batches
// One 1024-thread block, one slot per thread (R <= 1024).  Shared memory:
// cnt[32 warps][E] per-warp per-expert counts, turned into per-warp bases.
__global__ void __launch_bounds__(1024) route_small_kernel(const int64_t *__restrict__ topk_idx, int R, int k, int E,
                                                           int chunk_rows, int side, int *__restrict__ count,
                                                           int *__restrict__ offset, int *__restrict__ chunk_base,
                                                           int4 *__restrict__ chunks, int4 *__restrict__ chunks_s,
                                                           int *__restrict__ perm,
                                                           int *__restrict__ inv, int4 *__restrict__ rowinfo,
                                                           int *__restrict__ hdr, int32_t *__restrict__ expert_stats) {
    extern __shared__ int cnt[];
    __shared__ int s_warp[32];
    __shared__ int s_off[kMaxExperts], s_cbase[kMaxExperts];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    pdl_wait();
    pdl_trigger();
    for (int i = tid; i < 32 * E; i += 1024) cnt[i] = 0;
    __syncthreads();
    bool valid = false;
    int e = 0;
    if (tid < R) {
        const int64_t v = __ldcg(topk_idx + tid);
        valid = v >= 0 && v < E;
        e = valid ? int(v) : 0;
    }
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, valid ? unsigned(e) : 0xFFFFFFFFu);
    const int rank_w = __popc(peers & ((1u << lane) - 1u));
    if (valid && rank_w == 0) cnt[warp * E + e] = __popc(peers);
    const int nbad = __syncthreads_count(tid < R && !valid);
    // per expert: per-warp exclusive bases and the total
    int c = 0;
    if (tid < E)
        for (int w = 0; w < 32; ++w) {
            const int x = cnt[w * E + tid];
            cnt[w * E + tid] = c;
            c += x;
        }
    const bool s = tid < E && on_side(side, c);
    const int off = block_exclusive_scan(tid < E ? c : 0, s_warp);
    const int cbase = block_exclusive_scan(tid < E && !s ? (c + chunk_rows - 1) / chunk_rows : 0, s_warp);
    const int sbase = block_exclusive_scan(s && c > 0 ? 1 : 0, s_warp);
    if (tid < E) {
        s_off[tid] = off;
        s_cbase[tid] = s ? (kSideChunkBit | sbase) : cbase;
        write_expert_meta(tid, E, c, off, cbase, sbase, side, chunk_rows, count, offset, chunk_base, chunks,
                          chunks_s, hdr, expert_stats);
    }
    __syncthreads();
    if (tid < R) {
        if (valid) {
            const int local = cnt[warp * E + e] + rank_w;
            const int pos = s_off[e] + local;
            perm[pos] = tid;
            inv[tid] = pos;
            rowinfo[pos] = row_info(tid / k, s_cbase[e], local, chunk_rows);
        } else {
            inv[tid] = -1;
        }
    }
    if (tid == 0) {
        hdr[kHdrDropped] = nbad;
        hdr[kHdrError] = nbad ? kDevErrBadRouting : 0;
        hdr[kHdrTimeoutWhere] = 0;
    }
    for (int i = tid; i < 2 * kHdrSplitWords; i += blockDim.x) hdr[kHdrSplitCnt1 + i] = 0;
}

// ------------------------------------------------------------------ large batches
__global__ void __launch_bounds__(kRouteBlock) route_count_kernel(const int64_t *__restrict__ topk_idx, int R,
                                                                  int E, int *__restrict__ hist,
                                                                  int *__restrict__ lrank, int *__restrict__ bad) {
    extern __shared__ int cnt[];  // [kRouteBlock / 32][E]
    constexpr int kWarps = kRouteBlock / 32;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    pdl_wait();
    pdl_trigger();
    for (int i = tid; i < kWarps * E; i += kRouteBlock) cnt[i] = 0;
    __syncthreads();

    const int64_t s = int64_t(blockIdx.x) * kRouteBlock + tid;
    bool valid = false;
    int e = 0;
    if (s < R) {
        const int64_t v = __ldcg(topk_idx + s);
        valid = v >= 0 && v < E;
        e = valid ? int(v) : 0;
    }
    // rank among this warp's earlier lanes routed to the same expert
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, valid ? unsigned(e) : 0xFFFFFFFFu);
    const int rank_w = __popc(peers & ((1u << lane) - 1u));
    if (valid && rank_w == 0) cnt[warp * E + e] = __popc(peers);
    __syncthreads();
    if (valid) {
        int r = rank_w;
        for (int w = 0; w < warp; ++w) r += cnt[w * E + e];
        lrank[s] = r;
    }
    for (int x = tid; x < E; x += kRouteBlock) {
        int sum = 0;
        for (int w = 0; w < kWarps; ++w) sum += cnt[w * E + x];
        hist[size_t(x) * gridDim.x + blockIdx.x] = sum;  // expert-major
    }
    const int nbad = __syncthreads_count(s < R && !valid);
    if (tid == 0) bad[blockIdx.x] = nbad;
}

// One block per expert: exclusive prefix over the routing blocks of that
// expert's counts (in place, expert-major) and the expert's total.
__global__ void __launch_bounds__(1024) route_colscan_kernel(int *__restrict__ hist, int nb, int *__restrict__ count) {
    __shared__ int s_warp[32];
    __shared__ int s_carry;
    pdl_wait();
    pdl_trigger();
    const int e = blockIdx.x;
    int *row = hist + size_t(e) * nb;
    if (threadIdx.x == 0) s_carry = 0;
    __syncthreads();
    for (int b0 = 0; b0 < nb; b0 += blockDim.x) {
        const int b = b0 + threadIdx.x;
        const int v = b < nb ? __ldcg(row + b) : 0;
        const int ex = block_exclusive_scan(v, s_warp);
        const int carry = s_carry;
        if (b < nb) row[b] = carry + ex;
        __syncthreads();
        if (threadIdx.x == blockDim.x - 1) s_carry = carry + ex + v;
        __syncthreads();
    }
    if (threadIdx.x == 0) count[e] = s_carry;
}

// One block: offsets and chunk bases (scans over experts), chunk list,
// statistics, dropped count and error word.
__global__ void __launch_bounds__(1024) route_meta_kernel(const int *__restrict__ bad, int nb, int E, int chunk_rows,
                                                          int side, int *__restrict__ count, int *__restrict__ offset,
                                                          int *__restrict__ chunk_base, int4 *__restrict__ chunks,
                                                          int4 *__restrict__ chunks_s, int *__restrict__ hdr,
                                                          int32_t *__restrict__ expert_stats) {
    __shared__ int s_warp[32];
    __shared__ int s_bad;
    const int e = threadIdx.x;
    pdl_wait();
    pdl_trigger();
    const int c = e < E ? __ldcg(count + e) : 0;
    const bool s = e < E && on_side(side, c);
    const int off = block_exclusive_scan(c, s_warp);
    const int cbase = block_exclusive_scan(s ? 0 : (c + chunk_rows - 1) / chunk_rows, s_warp);
    const int sbase = block_exclusive_scan(s && c > 0 ? 1 : 0, s_warp);
    if (e < E)
        write_expert_meta(e, E, c, off, cbase, sbase, side, chunk_rows, count, offset, chunk_base, chunks, chunks_s,
                          hdr, expert_stats);
    if (threadIdx.x == 0) s_bad = 0;
    __syncthreads();
    int d = 0;
    for (int b = threadIdx.x; b < nb; b += blockDim.x) d += __ldcg(bad + b);
    if (d) atomicAdd(&s_bad, d);
    __syncthreads();
    if (threadIdx.x == 0) {
        hdr[kHdrDropped] = s_bad;
        hdr[kHdrError] = s_bad ? kDevErrBadRouting : 0;
        hdr[kHdrTimeoutWhere] = 0;
    }
    for (int i = threadIdx.x; i < 2 * kHdrSplitWords; i += blockDim.x) hdr[kHdrSplitCnt1 + i] = 0;
}

__global__ void __launch_bounds__(kRouteBlock) route_place_kernel(
    const int64_t *__restrict__ topk_idx, int R, int k, int E, int chunk_rows, const int *__restrict__ base,
    const int *__restrict__ lrank, const int *__restrict__ offset, const int *__restrict__ chunk_base,
    int *__restrict__ perm, int *__restrict__ inv, int4 *__restrict__ rowinfo) {
    pdl_wait();
    pdl_trigger();
    const int64_t s = int64_t(blockIdx.x) * kRouteBlock + threadIdx.x;
    if (s >= R) return;
    const int64_t v = __ldcg(topk_idx + s);
    if (v < 0 || v >= E) {
        inv[s] = -1;
        return;
    }
    const int e = int(v);
    const int pos = __ldcg(offset + e) + __ldcg(base + size_t(e) * gridDim.x + blockIdx.x) + __ldcg(lrank + s);
    perm[pos] = int(s);
    inv[s] = pos;
    const int local = pos - __ldcg(offset + e);
    rowinfo[pos] = row_info(int(s / k), __ldcg(chunk_base + e), local, chunk_rows);
}

// gather_kernel: one warp per task, a task being `seg_vec` 16-byte vectors of
// one routed row (the whole row for large batches; pieces of it when there are
// few rows, so that enough warps run); warps stride over the tasks.  A task's
// vectors move in batches of 32 lanes x kGatherVec, all loads of a batch issued
// before its stores; each vector goes to its column block's plane of the
// block-major destination [row_bytes/128][Rp][128] (8 lanes fill one 128-byte
// line).  The first task of a row also copies the row's scale words into the
// chunk's scale images: FP8 rows (row_bytes = H) have one word (4 groups of
// 32) per 128-byte block; NVFP4 rows (row_bytes = H/2) four (16 groups of 16),
// word w of a block going to image w of that block's images.
constexpr int kGatherThreads = 256;
constexpr int kGatherVec = 8;

__global__ void __launch_bounds__(kGatherThreads) gather_kernel(const int4 *__restrict__ rowinfo,
                                                                const int *__restrict__ offset, int E,
                                                                int row_bytes, int sf_words, int64_t Rp, int sf_bytes,
                                                                int sf_bytes_s, int segs, int seg_vec,
                                                                const uint8_t *__restrict__ x,
                                                                const uint8_t *__restrict__ x_sf,
                                                                uint8_t *__restrict__ xg, uint8_t *__restrict__ xg_sf,
                                                                uint8_t *__restrict__ xg_sf_s) {
    pdl_wait();
    pdl_trigger();
    constexpr int kWarps = kGatherThreads / 32;
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = int64_t(gridDim.x) * kWarps;
    const int64_t nrows = __ldcg(offset + E);  // dropped slots leave no row
    const int nvec = row_bytes / 16;
    const int KB = row_bytes / kTileK;  // 128-byte column blocks
    for (int64_t task = int64_t(blockIdx.x) * kWarps + (threadIdx.x >> 5); task < nrows * segs; task += nwarps) {
        const int64_t pos = task / segs;
        const int seg = int(task % segs);
        const int4 ri = __ldcg(rowinfo + pos);
        const uint4 *src = reinterpret_cast<const uint4 *>(x + int64_t(ri.x) * row_bytes);
        const int vend = (seg + 1) * seg_vec < nvec ? (seg + 1) * seg_vec : nvec;
        for (int base = seg * seg_vec; base < vend; base += 32 * kGatherVec) {
            uint4 v[kGatherVec];
#pragma unroll
            for (int i = 0; i < kGatherVec; ++i) {
                const int idx = base + i * 32 + lane;
                if (idx < vend) v[i] = __ldcg(src + idx);
            }
#pragma unroll
            for (int i = 0; i < kGatherVec; ++i) {
                const int idx = base + i * 32 + lane;
                if (idx < vend) {
                    const int col = idx * 16;
                    *reinterpret_cast<uint4 *>(xg + (int64_t(col / kTileK) * Rp + pos) * kTileK + col % kTileK) = v[i];
                }
            }
        }
        if (seg != 0) continue;
        const uint32_t *sfs = reinterpret_cast<const uint32_t *>(x_sf + int64_t(ri.x) * KB * sf_words * 4);
        // the chunk's images in its list's region (side-list chunks: 32 rows)
        uint8_t *const sf_dst = ri.w ? xg_sf_s : xg_sf;
        const int img_bytes = ri.w ? sf_bytes_s : sf_bytes;
        for (int wi = lane; wi < KB * sf_words; wi += 32) {
            const int kb = wi / sf_words, img = wi % sf_words;
            uint8_t *blk = sf_dst + ((int64_t(ri.y) * KB + kb) * sf_words + img) * img_bytes;
            *reinterpret_cast<uint32_t *>(blk + act_sf_offset(ri.z, 0)) = __ldcg(sfs + wi);
        }
    }
}

cudaError_t launch_routing(const int64_t *topk_idx, int k, int E, uint8_t *ws, const WsLayout &L,
                           int32_t *expert_stats, cudaStream_t stream) {
    const int R = int(L.R);
    int *hdr = reinterpret_cast<int *>(ws);
    int *hist = reinterpret_cast<int *>(ws + L.off_hist);
    int *bad = reinterpret_cast<int *>(ws + L.off_bad);
    int *lrank = reinterpret_cast<int *>(ws + L.off_lrank);
    int *count = reinterpret_cast<int *>(ws + L.off_count);
    int *offset = reinterpret_cast<int *>(ws + L.off_offset);
    int *chunk_base = reinterpret_cast<int *>(ws + L.off_chunk_base);
    int4 *chunks = reinterpret_cast<int4 *>(ws + L.off_chunks);
    int4 *chunks_s = reinterpret_cast<int4 *>(ws + L.off_chunks_s);
    const int side = L.side ? 1 : 0;
    int *perm = reinterpret_cast<int *>(ws + L.off_perm);
    int *inv = reinterpret_cast<int *>(ws + L.off_inv);
    int4 *rowinfo = reinterpret_cast<int4 *>(ws + L.off_rowinfo);
    const int cr = L.chunk_rows;
    cudaError_t e;
    if (R <= kRouteSmallMax) {
        const size_t smem = size_t(32) * E * sizeof(int);
        e = set_max_dynamic_smem(reinterpret_cast<const void *>(route_small_kernel),
                                 32 * kMaxExperts * int(sizeof(int)));
        if (e != cudaSuccess) return e;
        e = launch_pdl(route_small_kernel, dim3(1), dim3(1024), smem, stream, topk_idx, R, k, E, cr, side, count,
                       offset, chunk_base, chunks, chunks_s, perm, inv, rowinfo, hdr, expert_stats);
    } else {
        const size_t cnt_smem = size_t(kRouteBlock / 32) * E * sizeof(int);
        e = launch_pdl(route_count_kernel, dim3(L.nb), dim3(kRouteBlock), cnt_smem, stream, topk_idx, R, E, hist,
                       lrank, bad);
        const int cs_threads = L.nb >= 1024 ? 1024 : (L.nb + 31) / 32 * 32;
        if (e == cudaSuccess)
            e = launch_pdl(route_colscan_kernel, dim3(E), dim3(cs_threads), 0, stream, hist, L.nb, count);
        if (e == cudaSuccess)
            e = launch_pdl(route_meta_kernel, dim3(1), dim3(1024), 0, stream, static_cast<const int *>(bad), L.nb, E,
                           cr, side, count, offset, chunk_base, chunks, chunks_s, hdr, expert_stats);
        if (e == cudaSuccess)
            e = launch_pdl(route_place_kernel, dim3(L.nb), dim3(kRouteBlock), 0, stream, topk_idx, R, k, E, cr, hist,
                           lrank, offset, chunk_base, perm, inv, rowinfo);
    }
    return e;
}

cudaError_t launch_route(const int64_t *topk_idx, const uint8_t *x, const uint8_t *x_sf, int T, int k, int E,
                         int H, uint8_t *ws, const WsLayout &L, int32_t *expert_stats, bool nvfp4,
                         cudaStream_t stream) {
    cudaError_t e = launch_routing(topk_idx, k, E, ws, L, expert_stats, stream);
    if (e != cudaSuccess) return e;
    const int R = int(L.R);
    const int *offset = reinterpret_cast<const int *>(ws + L.off_offset);
    const int4 *rowinfo = reinterpret_cast<const int4 *>(ws + L.off_rowinfo);
    // up to 4 blocks per SM, striding over (row, piece) tasks; rows are cut
    // into pieces of a multiple of 32 vectors until there are about that many
    // warps' worth of tasks
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t warps = int64_t(sms) * 4 * (kGatherThreads / 32);
    const int row_bytes = nvfp4 ? H / 2 : H;
    const int nvec = row_bytes / 16;
    const int max_segs = (nvec + 31) / 32;
    int64_t segs = (warps + R - 1) / (R > 0 ? R : 1);
    if (segs > max_segs) segs = max_segs;
    if (segs < 1) segs = 1;
    const int seg_vec = int((max_segs + segs - 1) / segs) * 32;  // vectors per piece, a multiple of 32
    const int nseg = (nvec + seg_vec - 1) / seg_vec;  // pieces per row with that size
    const int64_t want = (int64_t(R) * nseg + kGatherThreads / 32 - 1) / (kGatherThreads / 32);
    const int grid = int(want < int64_t(sms) * 4 ? want : int64_t(sms) * 4);
    return launch_pdl(gather_kernel, dim3(unsigned(grid > 0 ? grid : 1)), dim3(kGatherThreads), 0, stream,
                      static_cast<const int4 *>(rowinfo), static_cast<const int *>(offset), E, row_bytes,
                      nvfp4 ? kNvImages : 1, int64_t(L.Rp), act_sf_bytes(L.chunk_rows),
                      act_sf_bytes(kChunkRowsSmall), nseg, seg_vec, x, x_sf, ws + L.off_xg, ws + L.off_xg_sf,
                      ws + L.off_xg_sf_s);
}

}  // namespace moe
