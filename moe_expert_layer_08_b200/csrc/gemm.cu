// gemm.cu -- the grouped expert GEMMs of the MoE layer on sm_100a tensor cores
// (phases 2-4 of "Mega moe fusion with symmetric memory", Procedure step 5:
// GEMM1 (FP8 x FP4), fused SwiGLU, GEMM2; FP8 activations and FP4 weights go
// to the tensor cores undequantised and the accumulator is fp32, as its Key
// design points state).
//
// One persistent kernel per GEMM over work items (chunk, output tile): a chunk
// is up to 128 consecutive routed rows of one expert, an output tile is 128
// weight rows.  The operands are swapped so that the weight tile is the
// MMA's M = 128 side and the chunk's tokens are the N side (N = rows rounded up
// to 16), which keeps decode-sized chunks (1-2 tokens per expert) from padding
// to 128.  Per CTA, warp-specialised:
//   warp 0 (one thread): TMA producer.  Per 128-K stage: the weight packet
//     body(s) via a 3D tensor map whose 4-bit element type expands FP4 into
//     the 1-byte-per-element shared-memory form the f8f6f4 MMA reads, the
//     packet's 512 scale bytes and the chunk's activation scale block via bulk
//     copies, the chunk's FP8 rows via 16-row 2D boxes.  Weights are one-use
//     (L2 evict-first), activations are re-read by every tile (evict-last).
//   warp 1 (one thread): tcgen05.cp of the stage's scale blocks into TMEM,
//     then 4 tcgen05.mma.kind::mxf8f6f4.block_scale (K = 32 each) per
//     accumulator; tcgen05.commit releases the stage and, after the last
//     stage, hands the accumulator to the epilogue.
//   warps 2-5: epilogue, TMEM -> registers (thread = weight row, registers =
//     tokens).  GEMM1: h = silu(gate) * up, per-token amax over each 32-row
//     group (a warp) by a transposing butterfly, UE8M0 scale, FP8 codes
//     written row-major plus the scale block of the chunk in the layout GEMM2's
//     tcgen05.cp consumes.  GEMM2: Y rows as bf16.
// Every mbarrier wait is bounded; on timeout the kernel records the failure in
// the workspace error word and all roles leave their loops.
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

template <bool kGemm1>
struct GemmCfg {
    static constexpr int kNumA = kGemm1 ? 2 : 1;        // accumulators (gate, up) or (down)
    static constexpr int kStages = kGemm1 ? 4 : 6;
    static constexpr int kATile = kTileRows * kTileK;   // 16 KB: 128 rows x 128 one-byte elements
    static constexpr int kBTile = kChunkRows * kTileK;  // 16 KB: up to 128 token rows
    static constexpr int kStageTiles = kNumA * kATile + kBTile;
    static constexpr int kStageSf = (kNumA + 1) * kSfBlockBytes;
    static constexpr int kSmemTiles = kStages * kStageTiles;
    static constexpr int kSmemSf = kStages * kStageSf;
    static constexpr int kSmemMisc = 256;
    static constexpr int kSmemBytes = 1024 + kSmemTiles + kSmemSf + kSmemMisc;
    static constexpr int kAccCols = kNumA * kChunkRows;
    static constexpr int kSfCols = kStages * (kNumA + 1) * 4;
    static constexpr int kTmemCols = (kAccCols + kSfCols) <= 256 ? 256 : 512;
    static_assert(kAccCols + kSfCols <= kTmemCols, "TMEM budget");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct GemmArgs {
    const uint8_t *w_packets;  // transformed weights (for the scale blocks)
    const uint8_t *act_sf;     // activation scale blocks [chunk][K/128][512]
    const int4 *chunks;        // (expert, first row, rows, -)
    int *hdr;                  // workspace header (chunk count, error word)
    uint8_t *out_q;            // GEMM1: h codes [R, I]
    uint8_t *out_sf;           // GEMM1: h scale blocks [chunk][I/128][512]
    __nv_bfloat16 *out_y;      // GEMM2: Y [R, H]
    int K;                     // reduction length (H for GEMM1, I for GEMM2)
    int n_tiles;               // output tiles per expert (I/128 or H/128)
    int out_ld;                // row length of the output (I or H)
};

// After the call lane l holds max over the warp's lanes of a[l] (the input
// arrays are consumed): 31 shuffles instead of 32 five-step all-reduces.
__device__ __forceinline__ float warp_transpose_max(float (&a)[32], int lane) {
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) {
        const bool upper = (lane & s) != 0;
#pragma unroll
        for (int i = 0; i < s; ++i) {
            const float send = upper ? a[i] : a[i + s];
            const float recv = __shfl_xor_sync(0xFFFFFFFFu, send, s);
            const float keep = upper ? a[i + s] : a[i];
            a[i] = fmaxf(keep, recv);
        }
    }
    return a[0];
}

template <bool kGemm1>
__global__ void __launch_bounds__(192, 1)
    moe_gemm_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_act,
                    const GemmArgs args) {
    using C = GemmCfg<kGemm1>;
    constexpr int kNumA = C::kNumA, kStages = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *tiles = smem;
    uint8_t *sfs = tiles + C::kSmemTiles;
    uint64_t *full = reinterpret_cast<uint64_t *>(sfs + C::kSmemSf);
    uint64_t *empty = full + kStages;
    uint64_t *tmem_full = empty + kStages;
    uint64_t *tmem_empty = tmem_full + 1;
    uint64_t *mma_done = tmem_empty + 1;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(tmem_full, 1);
        mbar_init(tmem_empty, 4);
        mbar_init(mma_done, 1);
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

    const int n_tiles = args.n_tiles;
    const int num_items = args.hdr[kHdrNumChunks] * n_tiles;
    const int KB = args.K / kTileK;
    int *err = args.hdr;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------------ producer
            const uint64_t pol_w = policy_evict_first();
            const uint64_t pol_a = policy_evict_last();
            int stage = 0;
            uint32_t phase = 0;
            uint32_t filled = 0, fill_parity = 0;
            bool ok = true;
            for (int item = blockIdx.x; ok && item < num_items; item += gridDim.x) {
                const int c = item / n_tiles, tile = item % n_tiles;
                const int4 ch = args.chunks[c];
                const int nbox = (ch.z + kBoxRows - 1) / kBoxRows;
                const uint32_t bytes = kNumA * (kPacketBody + kPacketSf) + nbox * kBoxRows * kTileK + kSfBlockBytes;
                const int64_t pkt0 = (int64_t(ch.x) * n_tiles + tile) * KB * kNumA;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, err, 1)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = tiles + stage * C::kStageTiles;
                    uint8_t *sf = sfs + stage * C::kStageSf;
                    mbar_arrive_expect_tx(&full[stage], bytes);
#pragma unroll
                    for (int a = 0; a < kNumA; ++a) {
                        const int64_t pkt = pkt0 + int64_t(kb) * kNumA + a;
                        tma_load_3d(st + a * C::kATile, &tmap_w, &full[stage], 0, 0, int(pkt), pol_w);
                        bulk_load(sf + a * kSfBlockBytes, args.w_packets + pkt * kPacketBytes + kPacketBody,
                                  kSfBlockBytes, &full[stage], pol_w);
                    }
                    for (int j = 0; j < nbox; ++j)
                        tma_load_2d(st + kNumA * C::kATile + j * kBoxRows * kTileK, &tmap_act, &full[stage],
                                    kb * kTileK, ch.y + j * kBoxRows, pol_a);
                    bulk_load(sf + kNumA * kSfBlockBytes, args.act_sf + (int64_t(c) * KB + kb) * kSfBlockBytes,
                              kSfBlockBytes, &full[stage], pol_a);
                    filled |= 1u << stage;
                    fill_parity = (fill_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // Every issued copy must have landed before the CTA may exit.
            for (int s = 0; s < kStages; ++s) {
                if (!(filled >> s & 1u)) continue;
                const uint32_t par = (fill_parity >> s) & 1u;
                const unsigned long long t0 = global_timer_ns();
                while (!mbar_try_wait(&full[s], par) && global_timer_ns() - t0 < kWaitTimeoutNs) {
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------------------ MMA issuer
            int stage = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int item = blockIdx.x; ok && item < num_items; item += gridDim.x) {
                const int4 ch = args.chunks[item / n_tiles];
                const uint32_t n = uint32_t((ch.z + kBoxRows - 1) / kBoxRows * kBoxRows);
                if (!mbar_wait(tmem_empty, acc_phase ^ 1u, abort_flag, err, 2)) break;
                tc_fence_after();
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&full[stage], phase, abort_flag, err, 3)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint8_t *st = tiles + stage * C::kStageTiles;
                    const uint8_t *sf = sfs + stage * C::kStageSf;
                    const uint32_t sf_col = tmem + C::kAccCols + stage * (kNumA + 1) * 4;
#pragma unroll
                    for (int a = 0; a <= kNumA; ++a)
                        tc_cp_sf(sf_col + a * 4, smem_desc_sf(smem_u32(sf + a * kSfBlockBytes)));
                    const uint64_t bdesc = smem_desc_sw128(smem_u32(st + kNumA * C::kATile));
#pragma unroll
                    for (int ks = 0; ks < kTileK / 32; ++ks) {
                        const uint32_t idesc = idesc_mxf8f6f4(n, uint32_t(ks));
#pragma unroll
                        for (int a = 0; a < kNumA; ++a) {
                            const uint64_t adesc = smem_desc_sw128(smem_u32(st + a * C::kATile));
                            // +32 bytes of K per step inside the 128-byte swizzled row
                            tc_mma_mxf8f6f4(tmem + a * kChunkRows, adesc + uint64_t(2 * ks),
                                            bdesc + uint64_t(2 * ks), idesc, sf_col + a * 4, sf_col + kNumA * 4,
                                            (kb | ks) != 0 ? 1u : 0u);
                        }
                    }
                    tc_commit(&empty[stage]);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit(tmem_full);
                acc_phase ^= 1u;
            }
            // All issued MMAs must be finished before TMEM is released.
            tc_commit(mma_done);
            const unsigned long long t0 = global_timer_ns();
            while (!mbar_try_wait(mma_done, 0) && global_timer_ns() - t0 < kWaitTimeoutNs) {
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- epilogue
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const uint32_t lane_base = uint32_t(q * 32) << 16;
        uint32_t acc_phase = 0;
        for (int item = blockIdx.x; item < num_items; item += gridDim.x) {
            const int c = item / n_tiles, tile = item % n_tiles;
            const int4 ch = args.chunks[c];
            if (!mbar_wait(tmem_full, acc_phase, abort_flag, err, 4)) break;
            tc_fence_after();
            const int ncb = (ch.z + 31) / 32;
            const int row_out = tile * kTileRows + q * 32 + lane;  // this thread's output column
            for (int cb = 0; cb < ncb; ++cb) {
                uint32_t g[32];
                tmem_ld_32x32(tmem + lane_base + uint32_t(cb * 32), g);
                if constexpr (kGemm1) {
                    uint32_t u[32];
                    tmem_ld_32x32(tmem + lane_base + uint32_t(kChunkRows + cb * 32), u);
                    tmem_ld_wait();
                    float h[32], a[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float gv = __uint_as_float(g[j]);
                        const float uv = __uint_as_float(u[j]);
                        h[j] = gv / (1.0f + expf(-gv)) * uv;
                        a[j] = fabsf(h[j]);
                    }
                    // lane l: amax of token cb*32+l over this warp's 32 rows of h
                    const float amax = warp_transpose_max(a, lane);
                    const int e = scale_exponent<true>(amax);
                    const float mult = exp2_neg(e);
                    const int tok = cb * 32 + lane;
                    if (tok < ch.z)
                        args.out_sf[(int64_t(c) * n_tiles + tile) * kSfBlockBytes + sf_block_offset(tok, q)] =
                            uint8_t(e + 127);
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float mj = __shfl_sync(0xFFFFFFFFu, mult, j);
                        const uint32_t code = to_e4m3(h[j] * mj);
                        if (cb * 32 + j < ch.z)
                            args.out_q[int64_t(ch.y + cb * 32 + j) * args.out_ld + row_out] = uint8_t(code);
                    }
                } else {
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (cb * 32 + j < ch.z)
                            args.out_y[int64_t(ch.y + cb * 32 + j) * args.out_ld + row_out] =
                                __float2bfloat16_rn(__uint_as_float(g[j]));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tmem_empty);
            acc_phase ^= 1u;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
}

template <bool kGemm1>
static cudaError_t launch_gemm_t(const CUtensorMap &tmap_w, const CUtensorMap &tmap_act, const GemmArgs &args,
                                 int grid, cudaStream_t stream) {
    using C = GemmCfg<kGemm1>;
    static int configured_for = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_for != dev) {
        const cudaError_t e = cudaFuncSetAttribute(moe_gemm_kernel<kGemm1>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
        if (e != cudaSuccess) return e;
        configured_for = dev;
    }
    moe_gemm_kernel<kGemm1><<<grid, 192, C::kSmemBytes, stream>>>(tmap_w, tmap_act, args);
    return cudaGetLastError();
}

cudaError_t launch_gemm(bool gemm1, const CUtensorMap &tmap_w, const CUtensorMap &tmap_act,
                        const uint8_t *w_packets, uint8_t *ws, const WsLayout &L, int H, int I, int grid,
                        cudaStream_t stream) {
    GemmArgs a{};
    a.w_packets = w_packets;
    a.chunks = reinterpret_cast<const int4 *>(ws + L.off_chunks);
    a.hdr = reinterpret_cast<int *>(ws);
    if (gemm1) {
        a.act_sf = ws + L.off_xg_sf;
        a.out_q = ws + L.off_hq;
        a.out_sf = ws + L.off_hq_sf;
        a.K = H;
        a.n_tiles = I / kTileRows;
        a.out_ld = I;
        return launch_gemm_t<true>(tmap_w, tmap_act, a, grid, stream);
    }
    a.act_sf = ws + L.off_hq_sf;
    a.out_y = reinterpret_cast<__nv_bfloat16 *>(ws + L.off_y);
    a.K = I;
    a.n_tiles = H / kTileRows;
    a.out_ld = H;
    return launch_gemm_t<false>(tmap_w, tmap_act, a, grid, stream);
}

}  // namespace moe
