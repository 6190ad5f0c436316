// shared.cu -- the BF16 shared expert (DeepGEMM PR #416: an optional dense
// expert that runs on every token beside the routed experts, bf16 input,
// weights and output; its test body defines the computation):
//   gate, up = bf16(x . L1^T)   (L1 rows 0..SI-1 gate, SI..2SI-1 up)
//   h        = bf16(act(gate, up))           (SwiGLU or SiTU)
//   y        = bf16(h . L2^T)
// Two persistent kernels, GEMM1 (+ activation) and GEMM2, on sm_100a tensor
// cores (tcgen05.mma.kind::f16, bf16 x bf16 -> fp32 in TMEM).  A work item is
// (block of kN tokens, pair of 128-row weight tiles); items are token-block
// major, so the CTAs working at one time share a token block (L2-resident) and
// every weight tile is re-read from L2 by later blocks.  Operands come by TMA
// straight from the row-major bf16 tensors (64 elements = one 128-byte
// swizzled row per K block): no gather and no layout transform.  Per CTA:
// warp 0 loads the two weight tiles, warp 6 the token tile, warps 1 and 7
// issue the MMAs of tile 0 and 1, and warps 2-5 (and 8-11 with 128-token
// blocks) drain the double-buffered TMEM accumulators.  With fewer items than
// SMs each item's K is cut into parts (one work unit each) whose fp32 partials
// are added in part order: across a thread-block cluster through distributed
// shared memory when the item's parts fit one cluster, else through global
// memory by the part that finishes last.  Every wait is bounded (workspace
// error word, as in the routed layer).
#include <mutex>
#include <vector>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

// kN = tokens per block (32 up to 64 tokens, 64 up to 128, else 128): a stage
// holds the item's two 128-row weight tiles and the block's token tile of one
// 64-element K block; as many stages as fit (192-216 KB of shared memory).
template <int kN>
struct SharedCfg {
    static constexpr int kStages = kN == 128 ? 4 : (kN == 64 ? 5 : 6);
    static constexpr int kATile = kTileRows * kTileK;  // 16 KB: 128 rows x 64 bf16
    static constexpr int kBTile = kN * kTileK;
    static constexpr int kStageBytes = 2 * kATile + kBTile;
    static constexpr int kSmemMisc = 256;
    static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kSmemMisc;
    static constexpr int kAccCols = 2 * kN;  // one accumulator buffer: tile 0, tile 1
    static constexpr int kTmemCols = 4 * kN <= 128 ? 128 : (4 * kN <= 256 ? 256 : 512);
    static constexpr int kEpiWarps = kN == 128 ? 8 : 4;
    static constexpr int kThreads = 32 * (kEpiWarps == 8 ? 12 : 8);
    static_assert(4 * kN <= kTmemCols, "two accumulator buffers");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
    static_assert(kBTile % 1024 == 0, "swizzle atoms");
    static_assert(8 * (2 * kStages + 8) + 12 <= kSmemMisc, "barriers and flags");
};

// K-split partial sums: one unit holds a part's fp32 accumulators of both
// tiles of its item, [tile][token][128 rows]; the scratch holds 256 units of
// 32-token blocks (8 MiB), 256 of 64-token blocks (16 MiB) or 160 of
// 128-token blocks (20 MiB), and no split needs more (about one unit per SM)
template <int kN>
constexpr int kSharedPartUnitFloats = 2 * kN * kTileRows;
constexpr int kSharedMaxUnits32 = 256;
constexpr int kSharedMaxUnits64 = 256;
constexpr int kSharedMaxUnits128 = 160;
// the most parts of one item that run as a thread-block cluster (above 8 the
// cluster size is non-portable: used where the device can hold the clusters),
// and how many parts the split may drop so that its clusters fit at once
constexpr int kSharedMaxClusterParts = 16;
constexpr int kSharedClusterShrink = 2;
static_assert(kSharedMaxUnits32 / 2 <= kHdrSplitWords && kSharedMaxUnits64 / 2 <= kHdrSplitWords &&
                  kSharedMaxUnits128 / 2 <= kHdrSplitWords,
              "a split item's counter in the header");

struct SharedArgs {
    int T;             // tokens
    int K;             // reduction length (SH for GEMM1, SI for GEMM2)
    int n_tiles;       // 128-row output tiles (GEMM1: SI / 128 per half, GEMM2: SH / 128)
    int n_items;       // tile pairs per token block
    int second_row;    // GEMM1: row of the up tile relative to the gate tile (SI); GEMM2: 128
    int out_ld;        // row length of the output (SI or SH)
    __nv_bfloat16 *out;
    int *hdr;          // workspace header (error word)
    int split;         // K parts per item (1: none)
    int cluster;       // split: 1 = each item's parts are one thread-block cluster (part = rank,
                       // one unit per CTA) that add their partials through distributed shared memory
    float *part;       // split: fp32 partial accumulators [unit][tile][kN tokens][128 rows]
    int *cnt;          // split: per item, parts finished (the last resets it)
    int *cnt_clear;    // the other GEMM's split counters (kHdrSplitWords), zeroed here
    int clear_err;     // GEMM1: zero the error word of this call
    int act_kind;      // GEMM1: MOE_ACT_SWIGLU or MOE_ACT_SITU
    float beta, inv_beta, lbeta, inv_lbeta;
};

__device__ __forceinline__ float bf16_round_f(float v) { return __bfloat162float(__float2bfloat16_rn(v)); }

// Every thread of every CTA of the cluster: shared-memory writes before it are
// visible to the cluster's CTAs after it.
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// The shared-memory address `saddr` of this CTA mapped into cluster CTA `rank`.
__device__ __forceinline__ uint32_t cluster_map(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}

template <bool kGemm1, int kN, bool kSplit>
__global__ void __launch_bounds__(SharedCfg<kN>::kThreads, 1)
    shared_gemm_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_act,
                       const SharedArgs args) {
    using C = SharedCfg<kN>;
    constexpr int kStages = C::kStages;
    static_assert(!kSplit || kSharedPartUnitFloats<kN> * 4 <= kStages * C::kStageBytes,
                  "a part's partials fit the operand ring (cluster mode)");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *tiles = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(tiles + kStages * C::kStageBytes);
    uint64_t *empty = full + kStages;
    uint64_t *tmem_full = empty + kStages;   // [2]
    uint64_t *tmem_empty = tmem_full + 2;    // [2]
    uint64_t *mma_done = tmem_empty + 2;     // [2]
    uint64_t *epi_bar = mma_done + 2;        // split: the epilogue warps' partials written
    uint64_t *epi_go = epi_bar + 1;          // split: the finishing decision taken
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(epi_go + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
    volatile int *epi_last = abort_flag + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool is_epi = (warp >= 2 && warp <= 5) || (C::kEpiWarps == 8 && warp >= 8);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 2);   // weight producer + token producer
            mbar_init(&empty[s], 2);  // both issuers
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tmem_full[b], 2);
            mbar_init(&tmem_empty[b], C::kEpiWarps);
            mbar_init(&mma_done[b], 1);
        }
        mbar_init(epi_bar, C::kEpiWarps);
        mbar_init(epi_go, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmap_w);
        prefetch_tmap(&tmap_act);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    // GEMM2's weights do not depend on GEMM1: its weight producer fills the
    // ring before GEMM1 has finished; every other access to memory written by
    // earlier kernels comes after pdl_wait
    if (kGemm1 || warp != 0) pdl_wait();
    if (blockIdx.x == 0 && warp == 1) {
        // The call's header upkeep, in place of a memset before the first
        // kernel (which would keep GEMM1 from starting under the previous
        // kernel's tail): GEMM1 clears the error word of this call, and each
        // GEMM clears the other's split counters (nonzero only after a call
        // that timed out). The kernel that used them last has completed
        // (griddepcontrol.wait above), and the next one to use them reads them
        // only after its own wait; the stores are fenced before the trigger
        // that lets the next kernel launch.
        for (int i = lane; i < kHdrSplitWords; i += 32) args.cnt_clear[i] = 0;
        if (args.clear_err && lane == 0) {
            args.hdr[kHdrError] = 0;
            args.hdr[kHdrTimeoutWhere] = 0;
        }
        __threadfence();
        __syncwarp();
    }
    if (threadIdx.x == 32) pdl_trigger();

    const int n_items = args.n_items, n_tiles = args.n_tiles;
    const int n_blocks = (args.T + kN - 1) / kN;
    const int num_items = n_blocks * n_items;
    const int KB = args.K / 64;  // K blocks of 64 bf16 (128 bytes)
    // work units: item u / split, K blocks [kb_lo(u), kb_hi(u)) of its K
    const int split = kSplit ? args.split : 1;
    const int num_units = num_items * split;
    auto kb_lo = [&](int u) { return (u % split) * KB / split; };
    auto kb_hi = [&](int u) { return (u % split + 1) * KB / split; };
    int *err = args.hdr;
    // rows of weight tile a of tile pair `it`
    auto tile_row = [&](int it, int a) {
        return kGemm1 ? it * kTileRows + a * args.second_row : (2 * it + a) * kTileRows;
    };

    if (warp == 0 || warp == 6) {
        if (lane == 0) {
            // -------------------------------------------------------- producers
            const bool weights = warp == 0;
            // weights are re-read by every token block (keep them in L2); a token
            // block is read by the CTAs of its items at about the same time
            const uint64_t pol = weights ? policy_evict_last() : policy_evict_first();
            int stage = 0;
            uint32_t phase = 0, filled = 0, fill_parity = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x) {
                const int item = u / split, blk = item / n_items, it = item % n_items;
                for (int kb = kb_lo(u); kb < kb_hi(u); ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, err, 11)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = tiles + stage * C::kStageBytes;
                    if (weights) {
                        // rows past the tensor (GEMM2's padded last pair) read as zeros
                        mbar_arrive_expect_tx(&full[stage], uint32_t(2 * C::kATile));
                        tma_load_2d(st, &tmap_w, &full[stage], kb * 64, tile_row(it, 0), pol);
                        tma_load_2d(st + C::kATile, &tmap_w, &full[stage], kb * 64, tile_row(it, 1), pol);
                    } else {
                        // tokens past T read as zeros
                        mbar_arrive_expect_tx(&full[stage], uint32_t(C::kBTile));
                        tma_load_2d(st + 2 * C::kATile, &tmap_act, &full[stage], kb * 64, blk * kN, pol);
                    }
                    filled |= 1u << stage;
                    fill_parity = (fill_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // every issued copy must have landed before the CTA may exit
            for (int s = 0; s < kStages; ++s) {
                if (!(filled >> s & 1u)) continue;
                const uint32_t par = (fill_parity >> s) & 1u;
                const unsigned long long t0 = global_timer_ns();
                while (!mbar_try_wait(&full[s], par) && global_timer_ns() - t0 < kWaitTimeoutNs) {
                }
            }
        }
        __syncwarp();
    } else if (warp == 1 || warp == 7) {
        if (lane == 0) {
            // -------------------------------------------------------- MMA issuer of tile a
            const int a = warp == 1 ? 0 : 1;
            int stage = 0, li = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < num_units; u += gridDim.x, ++li) {
                const int item = u / split, blk = item / n_items, it = item % n_items;
                const int k0 = kb_lo(u);
                const int rows = min(kN, args.T - blk * kN);
                const uint32_t n = uint32_t((rows + 15) / 16 * 16);
                const bool valid = kGemm1 || 2 * it + a < n_tiles;
                const int buf = li & 1;
                const uint32_t use = uint32_t(li >> 1) & 1u;
                if (!mbar_wait(&tmem_empty[buf], use ^ 1u, abort_flag, err, 12)) break;
                tc_fence_after();
                const uint32_t acc = tmem + uint32_t(buf * C::kAccCols + a * kN);
                for (int kb = k0; kb < kb_hi(u); ++kb) {
                    if (!mbar_wait(&full[stage], phase, abort_flag, err, 13)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (valid) {
                        const uint8_t *st = tiles + stage * C::kStageBytes;
                        const uint64_t adesc = smem_desc_sw128(smem_u32(st + a * C::kATile));
                        const uint64_t bdesc = smem_desc_sw128(smem_u32(st + 2 * C::kATile));
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            // 16 bf16 (32 bytes) of K per step inside the 128-byte swizzled row
                            tc_mma_bf16(acc, adesc + uint64_t(2 * ks), bdesc + uint64_t(2 * ks), idesc_bf16(n),
                                        (kb == k0 && ks == 0) ? 0u : 1u);
                    }
                    tc_commit(&empty[stage]);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit(&tmem_full[buf]);
            }
            // all issued MMAs must be finished before TMEM is released
            tc_commit(&mma_done[a]);
            const unsigned long long t0 = global_timer_ns();
            while (!mbar_try_wait(&mma_done[a], 0) && global_timer_ns() - t0 < kWaitTimeoutNs) {
            }
        }
        __syncwarp();
    } else if (is_epi) {
        // ------------------------------------------------------------ epilogue
        // thread = output column (weight row) q * 32 + lane of a tile,
        // registers = 32 consecutive tokens
        const int q = warp & 3;
        const int half = warp >= 8 ? 1 : 0;
        constexpr int kCbStep = C::kEpiWarps / 4;
        const uint32_t lane_base = uint32_t(q * 32) << 16;
        // GEMM1: h of kJ tokens of intermediate tile `it` from gate g and up u
        // (the linear layer's bf16 output, then the activation in fp32)
        auto finish1 = [&](const auto &g, const auto &u, int tok0, int nrows, int it) {
            constexpr int kJ = int(sizeof(g) / sizeof(g[0]));
            __nv_bfloat16 *hb = args.out + int64_t(tok0) * args.out_ld + it * kTileRows + q * 32 + lane;
            float h[kJ];
            if (args.act_kind == MOE_ACT_SWIGLU) {
#pragma unroll
                for (int j = 0; j < kJ; ++j) {
                    const float gv = bf16_round_f(__uint_as_float(g[j]));
                    const float uv = bf16_round_f(__uint_as_float(u[j]));
                    // silu(g) * u with the fast exponential and division, as in the
                    // routed experts' epilogue (0 where 1 + e^-g overflows: the limit)
                    h[j] = __fdividef(gv * uv, 1.0f + __expf(-gv));
                }
            } else {
#pragma unroll
                for (int j = 0; j < kJ; ++j) {
                    const float gv = bf16_round_f(__uint_as_float(g[j]));
                    const float uv = bf16_round_f(__uint_as_float(u[j]));
                    const float up = args.inv_lbeta != 0.0f ? args.lbeta * tanhf(uv * args.inv_lbeta) : uv;
                    h[j] = __fdividef(args.beta * tanhf(gv * args.inv_beta), 1.0f + __expf(-gv)) * up;
                }
            }
#pragma unroll
            for (int j = 0; j < kJ; ++j)
                if (j < nrows) hb[int64_t(j) * args.out_ld] = __float2bfloat16_rn(h[j]);
        };
        // GEMM2: y of kJ tokens of output tile `tile`
        auto finish2 = [&](const auto &v, int tok0, int nrows, int tile) {
            constexpr int kJ = int(sizeof(v) / sizeof(v[0]));
            __nv_bfloat16 *yb = args.out + int64_t(tok0) * args.out_ld + tile * kTileRows + q * 32 + lane;
#pragma unroll
            for (int j = 0; j < kJ; ++j)
                if (j < nrows) yb[int64_t(j) * args.out_ld] = __float2bfloat16_rn(__uint_as_float(v[j]));
        };
        int li = 0, nsplit = 0;
        for (int uu = blockIdx.x; uu < num_units; uu += gridDim.x, ++li) {
            const int item = uu / split, blk = item / n_items, it = item % n_items;
            const int rows = min(kN, args.T - blk * kN);
            const int buf = li & 1;
            const uint32_t use = uint32_t(li >> 1) & 1u;
            if (!mbar_wait(&tmem_full[buf], use, abort_flag, err, 14)) break;
            tc_fence_after();
            const uint32_t acc = tmem + lane_base + uint32_t(buf * C::kAccCols);
            if (split == 1) {
                const int ncb = (rows + 31) / 32;
                for (int cb = half; cb < ncb; cb += kCbStep) {
                    const int tok0 = blk * kN + cb * 32;
                    if constexpr (kGemm1) {
                        uint32_t g[32], u[32];
                        tmem_ld_32x32(acc + uint32_t(cb * 32), g);
                        tmem_ld_32x32(acc + uint32_t(kN + cb * 32), u);
                        tmem_ld_wait();
                        finish1(g, u, tok0, rows - cb * 32, it);
                    } else {
#pragma unroll 1
                        for (int a = 0; a < 2; ++a) {
                            if (2 * it + a >= n_tiles) break;
                            uint32_t v[32];
                            tmem_ld_32x32(acc + uint32_t(a * kN + cb * 32), v);
                            tmem_ld_wait();
                            finish2(v, tok0, rows - cb * 32, 2 * it + a);
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tmem_empty[buf]);
                continue;
            }
            // K part of an item: write this part's fp32 accumulators of the
            // block's real tokens (each warp its lane quarter of its column
            // blocks); the item's last part to finish adds the parts 0 ..
            // split-1 in that order and runs the epilogue, so the result does
            // not depend on which part ends last
            if constexpr (kSplit) {
                constexpr int kUnit = kSharedPartUnitFloats<kN>;
                const int ncb = (rows + 31) / 32;
                // cluster mode: the unit's MMAs are complete, so the operand ring
                // is free and holds this part's partials until the cluster reduces
                float *pu = (args.cluster ? reinterpret_cast<float *>(tiles) : args.part + size_t(uu) * kUnit) +
                            q * 32 + lane;
#pragma unroll 1
                for (int cb = half; cb < ncb; cb += kCbStep) {
#pragma unroll 1
                    for (int a = 0; a < 2; ++a) {
                        uint32_t v[32];
                        tmem_ld_32x32(acc + uint32_t(a * kN + cb * 32), v);
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (cb * 32 + j < rows) pu[(a * kN + cb * 32 + j) * kTileRows] = __uint_as_float(v[j]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tmem_empty[buf]);
                if (args.cluster) continue;  // reduced after the loop, across the cluster
                __threadfence();
                __syncwarp();
                if (lane == 0) mbar_arrive(epi_bar);
                if (warp == 2 && lane == 0) {
                    int last = 0;
                    if (mbar_wait(epi_bar, uint32_t(nsplit & 1), abort_flag, err, 15)) {
                        __threadfence();
                        last = atomicAdd(args.cnt + item, 1) == split - 1;
                        if (last) args.cnt[item] = 0;  // ready for the next launch
                        __threadfence();
                    }
                    *epi_last = last;
                    mbar_arrive(epi_go);
                }
                if (!mbar_wait(epi_go, uint32_t(nsplit & 1), abort_flag, err, 16)) break;
                ++nsplit;
                if (!*epi_last) continue;
                // the parts' sums, 8 tokens at a time, added in part order 0 ..
                // split-1 (the loads of four parts in flight together); then the
                // block's epilogue
                const float *p0 = args.part + size_t(item) * split * kUnit + q * 32 + lane;
#pragma unroll 1
                for (int jt = half * 32; jt < rows; jt += (jt & 31) == 24 ? 8 + 32 * (kCbStep - 1) : 8) {
                    const float *pj = p0 + jt * kTileRows;
                    uint32_t sv[2][8];
                    float s_[2][8];
#pragma unroll 1
                    for (int sp0 = 0; sp0 < split; sp0 += 4) {
                        float t[4][2][8];
#pragma unroll
                        for (int i = 0; i < 4; ++i)
#pragma unroll
                            for (int a = 0; a < 2; ++a)
#pragma unroll
                                for (int j = 0; j < 8; ++j)
                                    t[i][a][j] = sp0 + i < split ? __ldcg(pj + size_t(sp0 + i) * kUnit +
                                                                          (a * kN + j) * kTileRows)
                                                                 : 0.0f;
#pragma unroll
                        for (int i = 0; i < 4; ++i)
#pragma unroll
                            for (int a = 0; a < 2; ++a)
#pragma unroll
                                for (int j = 0; j < 8; ++j)
                                    if (sp0 + i == 0)
                                        s_[a][j] = t[i][a][j];
                                    else if (sp0 + i < split)
                                        s_[a][j] += t[i][a][j];
                    }
#pragma unroll
                    for (int a = 0; a < 2; ++a)
#pragma unroll
                        for (int j = 0; j < 8; ++j) sv[a][j] = __float_as_uint(s_[a][j]);
                    const int tok0 = blk * kN + jt;
                    if constexpr (kGemm1) {
                        finish1(sv[0], sv[1], tok0, rows - jt, it);
                    } else {
                        finish2(sv[0], tok0, rows - jt, 2 * it);
                        if (2 * it + 1 < n_tiles) finish2(sv[1], tok0, rows - jt, 2 * it + 1);
                    }
                }
            }
        }
        if constexpr (kSplit) {
            if (args.cluster) {
                __syncwarp();
                // one unit per CTA, part `rank` of item u / split: once every
                // part's partials are in its shared memory, the (rank, half)
                // warps take every nw-th 8-token group of the block, add the
                // parts' values in part order 0 .. split-1 (four parts' loads in
                // flight per round, the order of the global-memory path) and run
                // the epilogue on those 8 tokens
                cluster_sync_all();
                const int uu = int(blockIdx.x);
                if (uu < num_units && !*abort_flag) {
                    const int item = uu / split, blk = item / n_items, it = item % n_items;
                    const int rows = min(kN, args.T - blk * kN);
                    const int nw = split * kCbStep, me = (uu % split) * kCbStep + half;
                    const uint32_t p0 = smem_u32(reinterpret_cast<float *>(tiles) + q * 32 + lane);
#pragma unroll 1
                    for (int jt = me * 8; jt < rows; jt += nw * 8) {
                        uint32_t sv[2][8];
                        float s_[2][8];
#pragma unroll 1
                        for (int sp0 = 0; sp0 < split; sp0 += 4) {
                            float t[4][2][8];
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const uint32_t base = cluster_map(p0, uint32_t(sp0 + i < split ? sp0 + i : 0));
#pragma unroll
                                for (int a = 0; a < 2; ++a)
#pragma unroll
                                    for (int j = 0; j < 8; ++j)
                                        t[i][a][j] = sp0 + i < split
                                                         ? ld_cluster_f32(base + uint32_t((a * kN + jt + j) * kTileRows * 4))
                                                         : 0.0f;
                            }
#pragma unroll
                            for (int i = 0; i < 4; ++i)
#pragma unroll
                                for (int a = 0; a < 2; ++a)
#pragma unroll
                                    for (int j = 0; j < 8; ++j)
                                        if (sp0 + i == 0)
                                            s_[a][j] = t[i][a][j];
                                        else if (sp0 + i < split)
                                            s_[a][j] += t[i][a][j];
                        }
#pragma unroll
                        for (int a = 0; a < 2; ++a)
#pragma unroll
                            for (int j = 0; j < 8; ++j) sv[a][j] = __float_as_uint(s_[a][j]);
                        const int tok0 = blk * kN + jt;
                        if constexpr (kGemm1) {
                            finish1(sv[0], sv[1], tok0, rows - jt, it);
                        } else {
                            finish2(sv[0], tok0, rows - jt, 2 * it);
                            if (2 * it + 1 < n_tiles) finish2(sv[1], tok0, rows - jt, 2 * it + 1);
                        }
                    }
                }
                cluster_sync_all();  // the other parts are done reading this CTA's shared memory
            }
        }
    }
    // the warps outside the epilogue take the cluster's two barriers too
    if constexpr (kSplit)
        if (args.cluster && !is_epi) {
            cluster_sync_all();
            cluster_sync_all();
        }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
}

// Clusters of `cluster` CTAs of `kernel` (its dynamic shared memory already
// opted in) that can be resident at once on the current device, cached per
// (kernel, device, cluster size); 0 if the query fails.
static int max_active_clusters(const void *kernel, int cluster, int threads, int smem) {
    struct Memo {
        const void *kernel;
        int dev, cluster, n;
    };
    static std::mutex mu;
    static std::vector<Memo> memo;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> lock(mu);
    for (const Memo &m : memo)
        if (m.kernel == kernel && m.dev == dev && m.cluster == cluster) return m.n;
    if (cluster > 8 && cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
        (void)cudaGetLastError();
        memo.push_back({kernel, dev, cluster, 0});
        return 0;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(cluster * 16));
    cfg.blockDim = dim3(unsigned(threads));
    cfg.dynamicSmemBytes = size_t(smem);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = unsigned(cluster);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        n = 0;
    }
    memo.push_back({kernel, dev, cluster, n});
    return n;
}

template <bool kGemm1, int kN, bool kSplit>
static cudaError_t launch_shared_t(const CUtensorMap &tmap_w, const CUtensorMap &tmap_act, SharedArgs a, int items,
                                   cudaStream_t stream) {
    using C = SharedCfg<kN>;
    const void *kernel = reinterpret_cast<const void *>(shared_gemm_kernel<kGemm1, kN, kSplit>);
    const cudaError_t e = set_max_dynamic_smem(kernel, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    // K-split items whose parts fit one cluster each, every cluster resident
    // at once: the parts add their partials through distributed shared memory
    // (no global partials, fences or counters). Up to kSharedClusterShrink
    // fewer, longer parts are taken when that makes the clusters fit (on
    // B200 with the L2 flushed, T = 8: 37.8 -> 33.8 us per call, T = 32:
    // 48.1 -> 42.0 us, against the global-memory reduction with all parts);
    // otherwise the global path.
    a.cluster = 0;
    if (kSplit && a.split > 1)
        for (int s = a.split < kSharedMaxClusterParts ? a.split : kSharedMaxClusterParts;
             s >= 2 && s >= a.split - kSharedClusterShrink; --s)
            if (max_active_clusters(kernel, s, C::kThreads, C::kSmemBytes) >= items) {
                a.split = s;
                a.cluster = 1;
                break;
            }
    const int units = items * a.split;
    const int sms = num_sms();
    const int grid = a.cluster ? units : (units < sms ? (units > 0 ? units : 1) : sms);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(grid));
    cfg.blockDim = dim3(unsigned(C::kThreads));
    cfg.dynamicSmemBytes = size_t(C::kSmemBytes);
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = unsigned(a.cluster ? a.split : 1);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.cluster ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, shared_gemm_kernel<kGemm1, kN, kSplit>, tmap_w, tmap_act, a);
}

int shared_block_rows(int T) { return T <= kSharedTinyT ? 32 : T <= kSharedSmallT ? 64 : 128; }

size_t shared_part_bytes(int T) {
    const int kn = shared_block_rows(T);
    return kn == 32   ? size_t(kSharedMaxUnits32) * kSharedPartUnitFloats<32> * sizeof(float)
           : kn == 64 ? size_t(kSharedMaxUnits64) * kSharedPartUnitFloats<64> * sizeof(float)
                      : size_t(kSharedMaxUnits128) * kSharedPartUnitFloats<128> * sizeof(float);
}

cudaError_t launch_shared(bool gemm1, const CUtensorMap &tmap_w, const CUtensorMap &tmap_act, int T, int SH, int SI,
                          void *out, int *hdr, float *part, const moe_activation_t &act, cudaStream_t stream) {
    SharedArgs a{};
    a.T = T;
    a.hdr = hdr;
    a.part = part;
    // per item, reset by each item's last part; the other GEMM's counters are
    // cleared by this one (see the kernel)
    a.cnt = hdr + (gemm1 ? kHdrSplitCnt1 : kHdrSplitCnt2);
    a.cnt_clear = hdr + (gemm1 ? kHdrSplitCnt2 : kHdrSplitCnt1);
    a.clear_err = gemm1 ? 1 : 0;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.act_kind = act.kind;
    a.beta = act.beta;
    a.inv_beta = act.kind == MOE_ACT_SITU ? 1.0f / act.beta : 0.0f;
    a.lbeta = act.linear_beta;
    a.inv_lbeta = (act.kind == MOE_ACT_SITU && act.linear_beta > 0.0f) ? 1.0f / act.linear_beta : 0.0f;
    if (gemm1) {
        a.K = SH;
        a.n_tiles = SI / kTileRows;
        a.n_items = SI / kTileRows;
        a.second_row = SI;
        a.out_ld = SI;
    } else {
        a.K = SI;
        a.n_tiles = SH / kTileRows;
        a.n_items = (SH / kTileRows + 1) / 2;
        a.second_row = kTileRows;
        a.out_ld = SH;
    }
    const int kn = shared_block_rows(T);
    const int items = (T + kn - 1) / kn * a.n_items;
    // fewer items than SMs: cut each item's K into parts (at least four
    // 64-element K blocks each) so that about every SM works, as many units
    // as the partial-sum scratch holds
    const int sms = num_sms();
    const int max_units = kn == 32 ? kSharedMaxUnits32 : kn == 64 ? kSharedMaxUnits64 : kSharedMaxUnits128;
    a.split = 1;
    if (items < sms) {
        int s = sms / items;
        if (s > (a.K / 64) / 4) s = (a.K / 64) / 4;
        if (s > max_units / items) s = max_units / items;
        a.split = s > 1 ? s : 1;
    }
    // 32- and 64-token blocks: one kernel with and without a split; 128-token
    // blocks: the K-split epilogue only in the kernel that needs it
    if (kn == 32)
        return gemm1 ? launch_shared_t<true, 32, true>(tmap_w, tmap_act, a, items, stream)
                     : launch_shared_t<false, 32, true>(tmap_w, tmap_act, a, items, stream);
    if (kn == 64)
        return gemm1 ? launch_shared_t<true, 64, true>(tmap_w, tmap_act, a, items, stream)
                     : launch_shared_t<false, 64, true>(tmap_w, tmap_act, a, items, stream);
    if (a.split > 1)
        return gemm1 ? launch_shared_t<true, 128, true>(tmap_w, tmap_act, a, items, stream)
                     : launch_shared_t<false, 128, true>(tmap_w, tmap_act, a, items, stream);
    return gemm1 ? launch_shared_t<true, 128, false>(tmap_w, tmap_act, a, items, stream)
                 : launch_shared_t<false, 128, false>(tmap_w, tmap_act, a, items, stream);
}

}  // namespace moe
