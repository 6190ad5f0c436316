// route.cu -- routing (per-expert histogram, exclusive scan, stable
// permutation and its inverse, chunk list) and the local gather that replaces
// the cross-rank dispatch of the "Mega MoE" pipeline ("Mega moe fusion with
// symmetric memory", Procedure step 5, phase 1; the "gather-by-expert" step of
// What / Why).  Three launches, no host synchronisation:
//   1. route_count: per 256-slot block, per-expert counts and each slot's rank
//      among the block's earlier slots of the same expert;
//   2. route_scan (one block): counts, offsets, per-block base positions,
//      the list of <=128-row chunks per expert, expert statistics, error word;
//   3. route_place_gather: perm / inv, then the FP8 rows of x copied into
//      permuted order and their UE8M0 scales into per-chunk 512-byte blocks in
//      the layout tcgen05.cp copies into TMEM.
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

__global__ void __launch_bounds__(kRouteBlock) route_count_kernel(const int64_t *__restrict__ topk_idx, int R,
                                                                  int E, int *__restrict__ hist,
                                                                  int *__restrict__ lrank, int *__restrict__ bad) {
    extern __shared__ int cnt[];  // [kRouteBlock / 32][E]
    constexpr int kWarps = kRouteBlock / 32;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < kWarps * E; i += kRouteBlock) cnt[i] = 0;
    __syncthreads();

    const int64_t s = int64_t(blockIdx.x) * kRouteBlock + tid;
    bool valid = false;
    int e = 0;
    if (s < R) {
        const int64_t v = topk_idx[s];
        valid = v >= 0 && v < E;
        e = valid ? int(v) : 0;
    }
    // rank among this warp's earlier lanes routed to the same expert
    const unsigned key = valid ? unsigned(e) : 0xFFFFFFFFu;
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, key);
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
        hist[size_t(blockIdx.x) * E + x] = sum;
    }
    const int nbad = __syncthreads_count(s < R && !valid);
    if (tid == 0) bad[blockIdx.x] = nbad;
}

// Exclusive scan of one int per thread over a 1024-thread block.
__device__ __forceinline__ int block_exclusive_scan(int v, int *s_warp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = s_warp[lane];
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

__global__ void __launch_bounds__(1024) route_scan_kernel(int *__restrict__ hist, const int *__restrict__ bad,
                                                          int nb, int E, int *__restrict__ count,
                                                          int *__restrict__ offset, int *__restrict__ chunk_base,
                                                          int4 *__restrict__ chunks, int *__restrict__ hdr,
                                                          int32_t *__restrict__ expert_stats) {
    __shared__ int s_warp[32];
    __shared__ int s_bad;
    const int e = threadIdx.x;
    int c = 0;
    if (e < E)
        for (int b = 0; b < nb; ++b) c += hist[size_t(b) * E + e];
    const int nch = (c + kChunkRows - 1) / kChunkRows;
    const int off = block_exclusive_scan(c, s_warp);
    const int cbase = block_exclusive_scan(nch, s_warp);
    if (e < E) {
        count[e] = c;
        offset[e] = off;
        chunk_base[e] = cbase;
        int run = off;  // per-block base position of this expert's slots
        for (int b = 0; b < nb; ++b) {
            const size_t ix = size_t(b) * E + e;
            const int h = hist[ix];
            hist[ix] = run;
            run += h;
        }
        for (int q = 0; q < nch; ++q)
            chunks[cbase + q] = make_int4(e, off + q * kChunkRows, min(kChunkRows, c - q * kChunkRows), 0);
        if (expert_stats) expert_stats[e] += c;
        if (e == E - 1) {
            offset[E] = off + c;
            chunk_base[E] = cbase + nch;
            hdr[kHdrNumChunks] = cbase + nch;
        }
    }
    if (threadIdx.x == 0) s_bad = 0;
    __syncthreads();
    int d = 0;
    for (int b = threadIdx.x; b < nb; b += blockDim.x) d += bad[b];
    if (d) atomicAdd(&s_bad, d);
    __syncthreads();
    if (threadIdx.x == 0) {
        hdr[kHdrDropped] = s_bad;
        hdr[kHdrError] = s_bad ? kDevErrBadRouting : 0;
        hdr[kHdrTimeoutWhere] = 0;
    }
}

__global__ void __launch_bounds__(kRouteBlock) route_place_gather_kernel(
    const int64_t *__restrict__ topk_idx, int R, int k, int E, int H, const int *__restrict__ base,
    const int *__restrict__ lrank, const int *__restrict__ offset, const int *__restrict__ chunk_base,
    int *__restrict__ perm, int *__restrict__ inv, const uint8_t *__restrict__ x, const uint8_t *__restrict__ x_sf,
    uint8_t *__restrict__ xg, uint8_t *__restrict__ xg_sf) {
    __shared__ int s_t[kRouteBlock], s_pos[kRouteBlock], s_chunk[kRouteBlock], s_rl[kRouteBlock];
    const int tid = threadIdx.x;
    const int64_t s = int64_t(blockIdx.x) * kRouteBlock + tid;
    int pos = -1, t = 0, chunk = 0, rl = 0;
    if (s < R) {
        const int64_t v = topk_idx[s];
        if (v >= 0 && v < E) {
            const int e = int(v);
            pos = base[size_t(blockIdx.x) * E + e] + lrank[s];
            perm[pos] = int(s);
            inv[s] = pos;
            t = int(s / k);
            const int local = pos - offset[e];
            chunk = chunk_base[e] + local / kChunkRows;
            rl = local % kChunkRows;
        } else {
            inv[s] = -1;
        }
    }
    s_t[tid] = t;
    s_pos[tid] = pos;
    s_chunk[tid] = chunk;
    s_rl[tid] = rl;
    __syncthreads();

    const int warp = tid >> 5, lane = tid & 31;
    const int nvec = H / 16;
    const int KB = H / kTileK;
    for (int j = warp; j < kRouteBlock; j += kRouteBlock / 32) {
        const int p = s_pos[j];
        if (p < 0) continue;
        const uint4 *src = reinterpret_cast<const uint4 *>(x + size_t(s_t[j]) * H);
        uint4 *dst = reinterpret_cast<uint4 *>(xg + size_t(p) * H);
        for (int v = lane; v < nvec; v += 32) dst[v] = __ldg(src + v);
        const uint32_t *sfs = reinterpret_cast<const uint32_t *>(x_sf + size_t(s_t[j]) * (H / 32));
        for (int kb = lane; kb < KB; kb += 32) {
            uint8_t *blk = xg_sf + (size_t(s_chunk[j]) * KB + kb) * kSfBlockBytes;
            *reinterpret_cast<uint32_t *>(blk + sf_block_offset(s_rl[j], 0)) = __ldg(sfs + kb);
        }
    }
}

cudaError_t launch_route(const int64_t *topk_idx, const uint8_t *x, const uint8_t *x_sf, int T, int k, int E,
                         int H, uint8_t *ws, const WsLayout &L, int32_t *expert_stats, cudaStream_t stream) {
    const int R = int(L.R);
    int *hdr = reinterpret_cast<int *>(ws);
    int *hist = reinterpret_cast<int *>(ws + L.off_hist);
    int *bad = reinterpret_cast<int *>(ws + L.off_bad);
    int *lrank = reinterpret_cast<int *>(ws + L.off_lrank);
    int *count = reinterpret_cast<int *>(ws + L.off_count);
    int *offset = reinterpret_cast<int *>(ws + L.off_offset);
    int *chunk_base = reinterpret_cast<int *>(ws + L.off_chunk_base);
    int4 *chunks = reinterpret_cast<int4 *>(ws + L.off_chunks);
    int *perm = reinterpret_cast<int *>(ws + L.off_perm);
    int *inv = reinterpret_cast<int *>(ws + L.off_inv);
    const size_t cnt_smem = size_t(kRouteBlock / 32) * E * sizeof(int);
    route_count_kernel<<<L.nb, kRouteBlock, cnt_smem, stream>>>(topk_idx, R, E, hist, lrank, bad);
    route_scan_kernel<<<1, 1024, 0, stream>>>(hist, bad, L.nb, E, count, offset, chunk_base, chunks, hdr,
                                              expert_stats);
    route_place_gather_kernel<<<L.nb, kRouteBlock, 0, stream>>>(topk_idx, R, k, E, H, hist, lrank, offset,
                                                                chunk_base, perm, inv, x, x_sf, ws + L.off_xg,
                                                                ws + L.off_xg_sf);
    return cudaGetLastError();
}

}  // namespace moe
