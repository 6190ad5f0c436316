// gemm.cu -- the grouped expert GEMMs of the MoE layer on sm_100a tensor cores
// (phases 2-4 of "Mega moe fusion with symmetric memory", Procedure step 5:
// GEMM1 (FP8 x FP4), fused SwiGLU, GEMM2; FP8 activations and FP4 weights go
// to the tensor cores undequantised and the accumulator is fp32, as its Key
// design points state).
//
// One persistent kernel per GEMM over work items (chunk, pair of 128-row
// weight tiles): a chunk is up to kN consecutive routed rows of one expert
// (32 for small batches, 160 for large ones).  The operands are swapped so
// that the weight tile is the MMA's M = 128 side and the chunk's tokens are
// the N side (N = rows rounded up to 16), which keeps decode-sized chunks (1-2
// tokens per expert) from padding to 128.  Per CTA, warp-specialised:
//   warp 0 (one thread): weight producer.  Per stage one 4D TMA box of the
//     item's two tiles (a 4-bit element type that expands FP4 into the
//     1-byte-per-element shared-memory form the f8f6f4 MMA reads) and one 2D
//     box of their 512-byte scale blocks; weights are one-use (L2 evict-first).
//   warp 6 (one thread): activation producer.  The chunk's FP8 rows, stored
//     K-block-major, as 3D boxes (32-row boxes, or one kN-row box for a nearly
//     full large chunk) and the chunk's scale images by a bulk copy; they are
//     re-read by every tile of the chunk (evict-last).  NVFP4 with large
//     chunks: warp 0 loads the activations too, and warp 6 copies each
//     stage's activation scale images into TMEM for both issuers.
//   warps 1 and 7 (and 8, 9 with K split; one thread each): MMA issuers, one
//     per tile (and K half): tcgen05.cp of the stage's scale images into TMEM,
//     then tcgen05.mma.kind::mxf8f6f4.block_scale (K = 32 each) or
//     kind::mxf4nvf4 (K = 64); tcgen05.commit releases the stage and, after
//     the item's last stage, hands the accumulator to the epilogue.
//   The weight producer's warp streams before the grid-dependency wait; a
//   side-list launch waits at its end instead of its start.
//   warps 2-5 (and 8-11 for large chunks): epilogue, TMEM -> registers (thread
//     = weight row, registers = 32 tokens).  GEMM1: h = silu(gate) * up (or
//     SiTU), per-token amax over each 32-row group (a warp) by a transposing
//     butterfly, the scale, FP8 (or NVFP4) codes written K-block-major plus the
//     chunk's scale images in the layout GEMM2's tcgen05.cp consumes.  GEMM2:
//     Y rows as bf16.
// Items are dealt round-robin; with 32-row chunks the items of an incomplete
// last round are split along K over the idle CTAs (plan_work below).
// Every mbarrier wait is bounded; on timeout the kernel records the failure in
// the workspace error word and all roles leave their loops.
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

// kN = the largest token chunk an item can hold (the MMA's N).  Every item
// owns two 128-row weight tiles that share the chunk's activations: GEMM1 the
// gate and up tiles of one intermediate block, GEMM2 two adjacent output
// tiles.  Each tile has its own accumulator and its own MMA-issuing warp, since
// every tcgen05.mma / tcgen05.cp costs a fixed issue slot whatever its N.
// Small-batch launches (kN = 32) take 256-K stages.
//
// kNv: the NVFP4 variant.  A "K block" is always 128 bytes of an operand row
// in shared memory: 128 FP8 elements (or 128 FP4 expanded to bytes) in the
// FP8 x FP4 path, 256 packed E2M1 elements in the NVFP4 path, so the tiles,
// boxes and swizzle are the same; NVFP4 has four scale images per K block
// (one per 64-K MMA step) instead of one, and 256-K stages throughout.
template <bool kGemm1, int kN, bool kNv = false>
struct GemmCfg {
    static constexpr bool kSmall = kN == kChunkRowsSmall;
    static constexpr int kNumA = 2;                     // weight tiles (accumulators, issuers) per item
    static constexpr int kKB = kNv ? 1 : (kSmall ? 2 : 1);  // K blocks per pipeline stage
    // issuers per tile: with 32-row chunks and two K blocks per stage, two
    // threads split each tile's K blocks (even / odd) into two accumulators
    // that the epilogue adds, halving the tcgen05 issue time per stage
    // (NVFP4 with 32-row chunks: the stage's four 64-K MMA steps, two per issuer)
    static constexpr int kKSplit = (kSmall && (kKB == 2 || kNv)) ? 2 : 1;
    static constexpr int kIssuers = kNumA * kKSplit;
    static constexpr int kStages = kNv ? (kSmall ? 5 : 3) : (kSmall ? 3 : 4);
    static constexpr int kATile = kTileRows * kTileK;   // 16 KB: 128 rows x 128 bytes
    static constexpr int kBTile = kN * kTileK;          // token rows x 128 bytes, per K block
    static constexpr int kStageTiles = kNumA * kKB * kATile + kKB * kBTile;
    static constexpr int kActSf = act_sf_bytes(kN);     // one activation scale image set (all rows)
    static constexpr int kSfbImages = kActSf / kSfBlockBytes;
    static constexpr int kImg = kNv ? kNvImages : 1;    // scale image sets per K block
    static constexpr int kStageSf = kImg * (kNumA * kKB * kSfBlockBytes + kKB * kActSf);
    static constexpr int kWTx = kNv ? kNvPacketBytes : kPacketBytes;  // copy bytes per weight packet
    static constexpr int kSmemTiles = kStages * kStageTiles;
    static constexpr int kSmemSf = kStages * kStageSf;
    static constexpr int kSmemMisc = 256;
    // GEMM2 with large chunks: each epilogue warp stages 1 KB of bf16 output in
    // shared memory and writes whole row pieces with 16-byte stores instead of
    // 32 two-byte stores per row block (no room with 32-row chunks)
    // epilogue warps: two per TMEM lane quarter (alternating 32-token column
    // blocks) for large chunks; one per quarter for 32-row chunks, which are a
    // single column block
    static constexpr int kEpiWarpsC = kSmall ? 4 : 8;
    static constexpr bool kStaged = !kSmall && !kGemm1;
    static constexpr int kEpiStage = kStaged ? kEpiWarpsC * 1024 : 0;
    static constexpr int kSmemBytes = 1024 + kSmemTiles + kSmemSf + kSmemMisc + kEpiStage;
    static constexpr int kAccCols = kNumA * kKSplit * kN;  // one accumulator buffer
    // per issuer and stage: its weight tile's and the activations' scale images;
    // NVFP4 keeps two such regions per issuer (not one per stage) to fit TMEM,
    // the issuer waiting for the MMAs two stages back before reusing one
    static constexpr int kSfColsIssuer = kNv ? (kImg / kKSplit) * (1 + kSfbImages) * 4
                                             : (kKB / kKSplit) * kImg * (1 + kSfbImages) * 4;
    static constexpr int kSfRegions = kNv ? 2 : kStages;
    // NVFP4 with large chunks: a tcgen05 instruction costs its issuing thread
    // a fixed time whatever its N, and a 256-K stage takes each issuer four
    // MMAs and twelve scale copies, so the chunk's eight activation images
    // leave the two MMA issuers: warp 6 copies them (the weight producer, warp
    // 0, also loads the activations) into one TMEM region per stage slot that
    // both issuers read; each issuer still copies its own tile's four images
    // into the same region.  (The FP8 x FP4 kernels, with three copies per
    // issuer and stage, measured no faster this way.)
    static constexpr bool kCopier = !kSmall && kNv;
    static constexpr int kSfColsSlot = kImg * kKB * (kNumA + kSfbImages) * 4;
    static constexpr int kSfCols = kCopier ? kStages * kSfColsSlot : kSfRegions * kIssuers * kSfColsIssuer;
    static constexpr int kAccBufs = (2 * kAccCols + kSfCols) <= 512 ? 2 : 1;
    static constexpr int kTmemUsed = kAccBufs * kAccCols + kSfCols;
    static constexpr int kTmemCols = kTmemUsed <= 32 ? 32 : kTmemUsed <= 64 ? 64 : kTmemUsed <= 128 ? 128
                                   : kTmemUsed <= 256 ? 256 : 512;
    static constexpr int kEpiWarps = kEpiWarpsC;
    // warps: 0 weight producer, 6 activation producer, 1 / 7 / (8, 9) issuers,
    // 2-5 / (8-11) epilogue
    static constexpr int kThreads = 32 * (kEpiWarps == 8 ? 12 : (kIssuers == 4 ? 10 : 8));
    // weight packets one TMA box moves: an item's two tiles are adjacent for
    // every K tile (gate/up for GEMM1, a tile pair for GEMM2)
    static constexpr int kBoxPackets = kNumA * kKB;
    static_assert(kTmemUsed <= 512, "TMEM budget");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
    static_assert(8 * (3 * kStages + 11) + 12 <= kSmemMisc, "barriers and flags");
    static_assert(!kCopier || (kNv && kKB == 1 && kKSplit == 1), "the copier's regions hold one K block per stage");
    static_assert(!kSmall || kN * kNumA * kTileRows == kPartUnitFloats, "split-unit partial size");
    static_assert(kBTile % 1024 == 0, "swizzle atoms");
    static_assert(kKB == 1 || kN == kActBoxRows, "one activation box per stage when a stage spans K blocks");
    static_assert(kEpiWarps == 8 || kN <= 32, "one epilogue warp per quarter covers one column block");
    static_assert(!(kEpiWarps == 8 && kIssuers == 4), "warps 8-11 are either epilogue or issuers");
};

// Shared-memory slot of weight tile a (0, 1) of K block b within a stage:
// the order in which the packets land (K tile major, tile minor).
__device__ __forceinline__ int a_slot(int a, int b) { return b * 2 + a; }

struct GemmArgs {
    // weight layout: tile packets (body and scale block of each tile together)
    // or row-major FP4 bodies with the scale blocks in a separate array
    int w_rowmajor;
    int w_rows_per_expert;     // row-major: body rows of one expert (2I for L1, H for L2)
    int w_item_rows;           // row-major: body rows one item steps (128 for L1, 256 for L2)
    int w_sf_x0;               // word offset of a scale block within a row of the scale map
    const uint8_t *act_sf;     // activation scale blocks [chunk][K/128][512]
    const int4 *chunks;        // (expert, first row, rows, -)
    int *hdr;                  // workspace header (chunk counts, error word)
    int chunks_word;           // header word holding this list's chunk count
    uint8_t *out_q;            // GEMM1: h codes [R, I]
    uint8_t *out_sf;           // GEMM1: h scale blocks [chunk][I/128][512]
    __nv_bfloat16 *out_y;      // GEMM2: Y [R, H]
    int K;                     // reduction length (H for GEMM1, I for GEMM2)
    int n_tiles;               // 128-row weight tiles per expert and half (GEMM1: I/128, GEMM2: H/128)
    int n_items;               // items per chunk (GEMM1: I/128, GEMM2: tile pairs)
    int out_ld;                // row length of the output (I or H)
    int rows;                  // row extent of the K-block-major FP8 operands
    float *part;               // 32-row chunks: fp32 partial accumulators of split units [unit][tile][32][128]
    int *split_cnt;            // per leftover item: split units finished (reset by the last)
    int act_kind;              // GEMM1: MOE_ACT_SWIGLU or MOE_ACT_SITU
    float beta, inv_beta;      // SiTU coefficients (inv_lbeta = 0: no linear coefficient)
    float lbeta, inv_lbeta;
    // 1: the previous kernel is the main list's launch of this GEMM, which writes
    // nothing this launch reads: wait for it at the end, not the start
    int overlap_prev;
};

// After the call lane l holds, over the 16 lanes of its half-warp, the max of
// a[l % 16] in ra and of a[16 + l % 16] in rb (the arrays are consumed): the
// transposing butterfly below without its stage across half-warps, on the two
// 16-token halves side by side.
__device__ __forceinline__ void halfwarp_transpose_max(float (&a)[32], int lane, float &ra, float &rb) {
#pragma unroll
    for (int s = 8; s >= 1; s >>= 1) {
        const bool upper = (lane & s) != 0;
#pragma unroll
        for (int i = 0; i < s; ++i) {
#pragma unroll
            for (int h = 0; h < 32; h += 16) {
                const float send = upper ? a[h + i] : a[h + i + s];
                const float recv = __shfl_xor_sync(0xFFFFFFFFu, send, s);
                const float keep = upper ? a[h + i + s] : a[h + i];
                a[h + i] = fmaxf(keep, recv);
            }
        }
    }
    ra = a[0];
    rb = a[16];
}

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

// Work of one CTA.  Items are dealt round-robin; with 32-row chunks the items
// of an incomplete last round ("leftover" items) are instead cut along K into
// `split` units of whole stages, one unit per CTA, so that the last round
// keeps most SMs streaming weights.  Each unit writes its fp32 partial
// accumulators; the last unit of an item to finish (a per-item counter) adds
// all partials in unit order and runs the epilogue.  No CTA waits for another.
struct WorkPlan {
    int n_whole;     // whole items: blockIdx.x + k * gridDim.x for k < n_whole
    int split;       // units per leftover item (0: no split)
    int first_left;  // first leftover item
    int unit;        // this CTA's unit (-1: none): item first_left + unit / split, part unit % split
};

__device__ __forceinline__ WorkPlan plan_work(int num_items, int n_steps, bool allow_split) {
    WorkPlan P;
    const int G = int(gridDim.x), b = int(blockIdx.x);
    int whole_end = num_items, split = 0;
    if (allow_split) {
        const int rem = num_items % G;
        if (rem > 0) {
            int S = (G < kMaxSplitUnits ? G : kMaxSplitUnits) / rem;
            if (S > n_steps) S = n_steps;
            if (S >= 2) {
                split = S;
                whole_end = num_items - rem;
            }
        }
    }
    P.n_whole = b < whole_end ? (whole_end - b + G - 1) / G : 0;
    P.split = split;
    P.first_left = whole_end;
    P.unit = (split && b < (num_items - whole_end) * split) ? b : -1;
    return P;
}

// Work wk of the plan: item and stage range [s0, s1).
__device__ __forceinline__ void work_of(const WorkPlan &P, int wk, int n_steps, int &item, int &s0, int &s1) {
    if (wk < P.n_whole) {
        item = int(blockIdx.x) + wk * int(gridDim.x);
        s0 = 0;
        s1 = n_steps;
    } else {
        const int part = P.unit % P.split;
        item = P.first_left + P.unit / P.split;
        s0 = part * n_steps / P.split;
        s1 = (part + 1) * n_steps / P.split;
    }
}

template <bool kGemm1, int kN, bool kNv>
__global__ void __launch_bounds__(GemmCfg<kGemm1, kN, kNv>::kThreads, 1)
    moe_gemm_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_wsf,
                    const __grid_constant__ CUtensorMap tmap_act, const __grid_constant__ CUtensorMap tmap_act_full,
                    const GemmArgs args) {
    using C = GemmCfg<kGemm1, kN, kNv>;
    constexpr int kNumA = C::kNumA, kKB = C::kKB, kStages = C::kStages, kBufs = C::kAccBufs;
    constexpr int kIssuers = C::kIssuers;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *tiles = smem;
    uint8_t *sfs = tiles + C::kSmemTiles;
    uint64_t *full = reinterpret_cast<uint64_t *>(sfs + C::kSmemSf);
    uint64_t *empty = full + kStages;
    uint64_t *tmem_full = empty + kStages;   // [2]
    uint64_t *tmem_empty = tmem_full + 2;    // [2]
    uint64_t *mma_done = tmem_empty + 2;     // [kIssuers]
    uint64_t *epi_bar = mma_done + 4;        // split unit: epilogue warps' partials written
    uint64_t *epi_go = epi_bar + 1;          // split unit: the finishing decision taken
    uint64_t *sf_ready = epi_go + 1;         // [kStages] large chunks: the stage's scale images in TMEM
    uint64_t *cp_done = sf_ready + kStages;  // large chunks: all of the copier's copies complete
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(cp_done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
    volatile int *epi_last = abort_flag + 1;
    uint8_t *epi_stage = reinterpret_cast<uint8_t *>(full) + C::kSmemMisc;  // [kEpiWarps][1024] (large chunks)

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 2);  // weight copies + activation copies
            mbar_init(&empty[s], kIssuers);
            mbar_init(&sf_ready[s], 1);
        }
        mbar_init(cp_done, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tmem_full[b], kIssuers);
            mbar_init(&tmem_empty[b], C::kEpiWarps);
        }
        for (int i = 0; i < kIssuers; ++i) mbar_init(&mma_done[i], 1);
        mbar_init(epi_bar, C::kEpiWarps);
        mbar_init(epi_go, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmap_w);
        prefetch_tmap(&tmap_wsf);
        prefetch_tmap(&tmap_act);
        prefetch_tmap(&tmap_act_full);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    // The weights depend on neither kernel before this one (GEMM1: the gather;
    // GEMM2: GEMM1), and the routing's chunk list had been written when that
    // kernel started (it waited for the routing before letting this one
    // launch), so the weight producer's warp streams its first stages before
    // waiting; every other access to memory written by earlier kernels comes
    // after pdl_wait.  The whole warp skips the wait: a lane waiting alone would
    // hold lane 0 at the warp's reconvergence.  (With the scale-copy warp,
    // warp 0 also loads the activations and waits.)
    // A side-list launch (after the main list's launch of the same GEMM) uses
    // nothing that launch writes: it starts at once, overlapping its tail, and
    // waits at its end instead, so that it completes after it (what the next
    // kernel's wait relies on).
    const bool early_weights = warp == 0 && !C::kCopier;
    if (!early_weights && !args.overlap_prev) pdl_wait();
    if (threadIdx.x == 32) pdl_trigger();

    const int n_tiles = args.n_tiles, n_items = args.n_items;
    const int num_items = __ldcg(args.hdr + args.chunks_word) * n_items;
    const int KB = args.K / (kNv ? kNvTileK : kTileK);  // K blocks of 128 operand bytes
    const int n_steps = (KB + kKB - 1) / kKB;  // pipeline stages per item
    const WorkPlan P = plan_work(num_items, n_steps, C::kSmall);
    const int n_works = P.n_whole + (P.unit >= 0 ? 1 : 0);
    int *err = args.hdr;

    // which MMA issuer this warp is (-1: none)
    const int issuer = warp == 1 ? 0 : warp == 7 ? 1 : (kIssuers == 4 && warp == 8) ? 2
                     : (kIssuers == 4 && warp == 9) ? 3 : -1;

    if (warp == 0 || (warp == 6 && !C::kCopier)) {
        if (lane == 0) {
            // ------------------------------------------------------------ producers
            // weight packets and their scale blocks (one box each per stage;
            // warp 0), the chunk's activation K blocks (one 3D box of kKB K
            // blocks x 32 rows per 32 rows) and their scale blocks (warp 6, or
            // warp 0 as well with large chunks)
            const bool weights = warp == 0, acts = C::kCopier || warp == 6;
            const uint64_t pol_w = policy_evict_first(), pol_a = policy_evict_last();
            int stage = 0;
            uint32_t phase = 0;
            uint32_t filled = 0, fill_parity = 0;
            bool ok = true;
            for (int wk = 0; ok && wk < n_works; ++wk) {
                int item, s0, s1;
                work_of(P, wk, n_steps, item, s0, s1);
                const int c = item / n_items, it = item % n_items;
                const int4 ch = __ldcg(args.chunks + c);
                const int nbox = (ch.z + kActBoxRows - 1) / kActBoxRows;
                // GEMM1: gate/up packets of tile `it`, interleaved per K tile;
                // GEMM2: tiles 2*it and 2*it+1 (the second may not exist)
                // packet group of the item: gate/up pair `it` (GEMM1) or tile pair `it` (GEMM2)
                const int groups = kGemm1 ? n_tiles : n_items;
                for (int step = s0; step < s1; ++step) {
                    const int kb0 = step * kKB;
                    const int nkb = min(kKB, KB - kb0);
                    if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, err, acts && !weights ? 5 : 1)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = tiles + stage * C::kStageTiles;
                    uint8_t *sf = sfs + stage * C::kStageSf;
                    if (weights) {
                        // a box always moves kBoxPackets packets (a last odd K
                        // block loads packets it then ignores)
                        mbar_arrive_expect_tx(&full[stage], uint32_t(kNumA * kKB * C::kWTx));
                        // 4D box (128 K, 128 rows, tile a, K block b) lands as slots b * 2 + a
                        const int pkt = int((int64_t(ch.x) * groups + it) * KB * 2 + int64_t(kb0) * 2);
                        if (kNv) {
                            // packed E2M1 bodies as bytes; scale images (128 words, image, packet)
                            tma_load_4d(st, &tmap_w, &full[stage], 0, 0, 0, pkt / 2, pol_w);
                            tma_load_3d(sf, &tmap_wsf, &full[stage], 0, 0, pkt, pol_w);
                        } else {
                            if (args.w_rowmajor)
                                tma_load_4d(st, &tmap_w, &full[stage], 0,
                                            ch.x * args.w_rows_per_expert + it * args.w_item_rows, 0, kb0, pol_w);
                            else
                                tma_load_4d(st, &tmap_w, &full[stage], 0, 0, 0, pkt / 2, pol_w);
                            tma_load_2d(sf, &tmap_wsf, &full[stage], args.w_sf_x0, pkt, pol_w);
                        }
                    }
                    if (acts) {
                        // the activation box always moves kKB K blocks (a K
                        // block past the end reads zeros); a nearly full large
                        // chunk takes one kN-row box instead of several 32-row ones
                        const bool one_box = !C::kSmall && ch.z > kN - 64;
                        const int rows_moved = one_box ? kN : nbox * kActBoxRows;
                        mbar_arrive_expect_tx(&full[stage],
                                              uint32_t(rows_moved * kKB * kTileK + nkb * C::kImg * C::kActSf));
                        uint8_t *bt = st + kNumA * kKB * C::kATile;
                        if (one_box) {
                            tma_load_3d(bt, &tmap_act_full, &full[stage], 0, ch.y, kb0, pol_a);
                        } else {
                            for (int j = 0; j < nbox; ++j)
                                tma_load_3d(bt + j * kActBoxRows * kTileK, &tmap_act, &full[stage], 0,
                                            ch.y + j * kActBoxRows, kb0, pol_a);
                        }
                        bulk_load(sf + C::kImg * kNumA * kKB * kSfBlockBytes,
                                  args.act_sf + (int64_t(c) * KB + kb0) * C::kImg * C::kActSf,
                                  nkb * C::kImg * C::kActSf, &full[stage], pol_a);
                    }
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
    } else if (C::kCopier && warp == 6) {
        if (lane == 0) {
            // ------------------------------------------------------------ scale copier
            // For every stage: once its data has landed, the chunk's activation
            // scale images of the four 64-K steps go to the stage slot's TMEM
            // region; the slot's previous MMAs are complete by then (the
            // producer refilled it after their commits).
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int wk = 0; ok && wk < n_works; ++wk) {
                int item, s0, s1;
                work_of(P, wk, n_steps, item, s0, s1);
                const int4 ch = __ldcg(args.chunks + item / n_items);
                const int sfb_images = (ch.z + 15) / 16 * 16 > 128 ? 2 : 1;
                for (int step = s0; step < s1; ++step) {
                    if (!mbar_wait(&full[stage], phase, abort_flag, err, 9)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint8_t *sfa = sfs + stage * C::kStageSf;
                    const uint32_t col = tmem + uint32_t(kBufs * C::kAccCols + stage * C::kSfColsSlot);
                    const uint8_t *sfb = sfa + kNumA * kNvImages * kSfBlockBytes;
                    const uint32_t colb = col + kNumA * kNvImages * 4;
#pragma unroll
                    for (int j = 0; j < kNvImages; ++j)
#pragma unroll
                        for (int im = 0; im < C::kSfbImages; ++im)
                            if (im < sfb_images)
                                tc_cp_sf(colb + (j * C::kSfbImages + im) * 4,
                                         smem_desc_sf(smem_u32(sfb + j * C::kActSf + im * kSfBlockBytes)));
                    tc_commit(&sf_ready[stage]);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // the copies must be complete before TMEM is released
            tc_commit(cp_done);
            const unsigned long long t0 = global_timer_ns();
            while (!mbar_try_wait(cp_done, 0) && global_timer_ns() - t0 < kWaitTimeoutNs) {
            }
        }
        __syncwarp();
    } else if (issuer >= 0) {
        if (lane == 0) {
            // ------------------------------------------------------------ MMA issuer
            // Issuer (a, h) owns weight tile a of every item and, for K split
            // h of kKSplit, its accumulator: the stage's K blocks b with
            // b % kKSplit == h (NVFP4: the stage's 64-K steps 2h and 2h + 1).
            const int a = issuer % kNumA, h = issuer / kNumA;
            int stage = 0;
            uint32_t phase = 0;
            int li = 0;        // items handled by this CTA so far
            int gstage = 0;    // stages consumed so far (all items)
            bool ok = true;
            for (int wk = 0; ok && wk < n_works; ++wk, ++li) {
                int item, s0, s1;
                work_of(P, wk, n_steps, item, s0, s1);
                const int4 ch = __ldcg(args.chunks + item / n_items);
                const int it = item % n_items;
                const bool valid = kGemm1 || 2 * it + a < n_tiles;  // GEMM2's last pair may hold one tile
                const uint32_t n = uint32_t((ch.z + 15) / 16 * 16);
                // activation scale images the MMAs read: one per 128 of the N rows
                const int sfb_images = int(n + 127) / 128;
                const int buf = li % kBufs;
                const uint32_t use = uint32_t(li / kBufs) & 1u;  // how often this buffer was used, mod 2
                if (!mbar_wait(&tmem_empty[buf], use ^ 1u, abort_flag, err, 2)) break;
                tc_fence_after();
                const uint32_t acc = tmem + uint32_t(buf * C::kAccCols + (h * kNumA + a) * kN);
                for (int step = s0; step < s1; ++step) {
                    const int kb0 = step * kKB;
                    const int nkb = min(kKB, KB - kb0);
                    if (!mbar_wait(&full[stage], phase, abort_flag, err, 3)) {
                        ok = false;
                        break;
                    }
                    if (C::kCopier && !mbar_wait(&sf_ready[stage], phase, abort_flag, err, 10)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (C::kCopier) {
                        // this stage slot's region: the A images of both tiles (this
                        // issuer copies its own four here), then the chunk's
                        // activation images (from the copier)
                        const uint8_t *st = tiles + stage * C::kStageTiles;
                        const uint32_t col = tmem + uint32_t(kBufs * C::kAccCols + stage * C::kSfColsSlot);
                        const uint64_t adesc = smem_desc_sw128(smem_u32(st + a * C::kATile));
                        const uint64_t bdesc = smem_desc_sw128(smem_u32(st + kNumA * C::kATile));
                        if (valid) {
                            const uint8_t *sfa = sfs + stage * C::kStageSf;
                            const uint32_t cola = col + a * kNvImages * 4, colb = col + kNumA * kNvImages * 4;
#pragma unroll
                            for (int j = 0; j < kNvImages; ++j)
                                tc_cp_sf(cola + j * 4, smem_desc_sf(smem_u32(sfa + (a * kNvImages + j) * kSfBlockBytes)));
#pragma unroll
                            for (int j = 0; j < kNvImages; ++j)
                                // 64 K (32 bytes) per step inside the 128-byte swizzled row, one image each
                                tc_mma_nvf4(acc, adesc + uint64_t(2 * j), bdesc + uint64_t(2 * j), idesc_nvf4(n),
                                            cola + j * 4, colb + j * C::kSfbImages * 4,
                                            (step == s0 && j == 0) ? 0u : 1u);
                        }
                    } else if (kNv && valid && gstage >= 2) {
                        // this issuer's scale region was last read by the MMAs of stage
                        // gstage - 2: their commit has completed that stage's `empty` phase
                        const int g2 = gstage - 2;
                        if (!mbar_wait(&empty[g2 % kStages], uint32_t(g2 / kStages) & 1u, abort_flag, err, 6)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                    }
                    if (C::kCopier) {
                    } else if (kNv && valid) {
                        // this issuer's MMA steps ks = h * kSteps .. (h + 1) * kSteps - 1
                        // of the four, each with its weight and activation scale image
                        constexpr int kSteps = kNvImages / C::kKSplit;
                        const uint8_t *st = tiles + stage * C::kStageTiles;
                        const uint8_t *sfa = sfs + stage * C::kStageSf;           // [tile][image][512]
                        const uint8_t *sfb = sfa + kNumA * kNvImages * kSfBlockBytes;  // [image][kActSf]
                        const uint8_t *bt = st + kNumA * C::kATile;
                        const uint32_t col = tmem + uint32_t(kBufs * C::kAccCols +
                                                             ((gstage & 1) * kIssuers + issuer) * C::kSfColsIssuer);
                        const uint32_t colb = col + kSteps * 4;
#pragma unroll
                        for (int j = 0; j < kSteps; ++j) {
                            const int sI = h * kSteps + j;
                            tc_cp_sf(col + j * 4, smem_desc_sf(smem_u32(sfa + (a * kNvImages + sI) * kSfBlockBytes)));
#pragma unroll
                            for (int im = 0; im < C::kSfbImages; ++im)
                                if (im < sfb_images)
                                    tc_cp_sf(colb + (j * C::kSfbImages + im) * 4,
                                             smem_desc_sf(smem_u32(sfb + sI * C::kActSf + im * kSfBlockBytes)));
                        }
                        const uint64_t adesc = smem_desc_sw128(smem_u32(st + a * C::kATile));
                        const uint64_t bdesc = smem_desc_sw128(smem_u32(bt));
#pragma unroll
                        for (int j = 0; j < kSteps; ++j) {
                            // 64 K (32 bytes) per step inside the 128-byte swizzled row, one image each
                            const int ks = h * kSteps + j;
                            tc_mma_nvf4(acc, adesc + uint64_t(2 * ks), bdesc + uint64_t(2 * ks), idesc_nvf4(n),
                                        col + j * 4, colb + j * C::kSfbImages * 4,
                                        (step == s0 && j == 0) ? 0u : 1u);
                        }
                    } else if (valid) {
                        const uint8_t *st = tiles + stage * C::kStageTiles;
                        const uint8_t *sfa = sfs + stage * C::kStageSf;
                        const uint8_t *sfb = sfa + kNumA * kKB * kSfBlockBytes;
                        const uint8_t *bt = st + kNumA * kKB * C::kATile;
                        uint32_t col =
                            tmem + uint32_t(kBufs * C::kAccCols + (stage * kIssuers + issuer) * C::kSfColsIssuer);
                        for (int b = 0; b < nkb; ++b) {
                            if (b % C::kKSplit != h) continue;
                            const int slot = a_slot(a, b);
                            // scale images of this K block into TMEM: weight tile, then activations
                            tc_cp_sf(col, smem_desc_sf(smem_u32(sfa + slot * kSfBlockBytes)));
                            const uint32_t sfb_col = col + 4;
#pragma unroll
                            for (int im = 0; im < C::kSfbImages; ++im)
                                if (im < sfb_images)
                                    tc_cp_sf(sfb_col + im * 4,
                                             smem_desc_sf(smem_u32(sfb + b * C::kActSf + im * kSfBlockBytes)));
                            const uint64_t adesc = smem_desc_sw128(smem_u32(st + slot * C::kATile));
                            const uint64_t bdesc = smem_desc_sw128(smem_u32(bt + b * C::kBTile));
#pragma unroll
                            for (int ks = 0; ks < kTileK / 32; ++ks) {
                                // +32 bytes of K per step inside the 128-byte swizzled row
                                tc_mma_mxf8f6f4(acc, adesc + uint64_t(2 * ks), bdesc + uint64_t(2 * ks),
                                                idesc_mxf8f6f4(n, uint32_t(ks)), col, sfb_col,
                                                (kb0 + b == s0 * kKB + h && ks == 0) ? 0u : 1u);
                            }
                            col += uint32_t((1 + C::kSfbImages) * 4);
                        }
                    }
                    tc_commit(&empty[stage]);
                    ++gstage;
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit(&tmem_full[buf]);
            }
            // All issued MMAs must be finished before TMEM is released.
            tc_commit(&mma_done[issuer]);
            const unsigned long long t0 = global_timer_ns();
            while (!mbar_try_wait(&mma_done[issuer], 0) && global_timer_ns() - t0 < kWaitTimeoutNs) {
            }
        }
        __syncwarp();
    } else if ((warp >= 2 && warp <= 5) || (C::kEpiWarps == 8 && warp >= 8)) {
        // ---------------------------------------------------------------- epilogue
        const int q = warp & 3;                 // TMEM lane quarter this warp may access
        const int half = warp >= 8 ? 1 : 0;     // which column blocks of the quarter it handles
        constexpr int kCbStep = C::kEpiWarps / 4;
        uint8_t *my_stage = epi_stage + (warp < 8 ? warp - 2 : warp - 4) * 1024;
        const uint32_t lane_base = uint32_t(q * 32) << 16;
        int li = 0;
        for (int wk = 0; wk < n_works; ++wk, ++li) {
            int item, s0, s1;
            work_of(P, wk, n_steps, item, s0, s1);
            const bool is_unit = wk >= P.n_whole;
            const int c = item / n_items, it = item % n_items;
            const int4 ch = __ldcg(args.chunks + c);
            const int buf = li % kBufs;
            const uint32_t use = uint32_t(li / kBufs) & 1u;
            if (!mbar_wait(&tmem_full[buf], use, abort_flag, err, 4)) break;
            tc_fence_after();
            const uint32_t acc = tmem + lane_base + uint32_t(buf * C::kAccCols);
            const int ncb = (ch.z + 31) / 32;
            // with K split, accumulator kNumA + a holds tile a's K blocks of
            // odd index, written when the stage range holds one (NVFP4: the
            // last two 64-K steps of every stage)
            const bool add_split = C::kKSplit == 2 && (kNv || s0 * kKB + 1 < min(s1 * kKB, KB));
            // GEMM2: fp32 words of token cb*32 + j of output tile 2 * it + a
            auto load_tile = [&](int a, int cb, uint32_t (&v)[32]) {
                tmem_ld_32x32(acc + uint32_t(a * kN + cb * 32), v);
                tmem_ld_wait();
                if (add_split) {
                    uint32_t v1[32];
                    tmem_ld_32x32(acc + uint32_t((kNumA + a) * kN + cb * 32), v1);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) + __uint_as_float(v1[j]));
                }
            };
            // GEMM1: gate and up accumulators of column block cb (K split: both halves added)
            auto load_gu = [&](int cb, uint32_t (&g)[32], uint32_t (&u)[32]) {
                tmem_ld_32x32(acc + uint32_t(cb * 32), g);
                tmem_ld_32x32(acc + uint32_t(kN + cb * 32), u);
                tmem_ld_wait();
                if (add_split) {
                    uint32_t g1[32], u1[32];
                    tmem_ld_32x32(acc + uint32_t(2 * kN + cb * 32), g1);
                    tmem_ld_32x32(acc + uint32_t(3 * kN + cb * 32), u1);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        g[j] = __float_as_uint(__uint_as_float(g[j]) + __uint_as_float(g1[j]));
                        u[j] = __float_as_uint(__uint_as_float(u[j]) + __uint_as_float(u1[j]));
                    }
                }
            };
            // h = act(gate, up) of 32 tokens of this lane's intermediate row
            auto activate = [&](const uint32_t (&g)[32], const uint32_t (&u)[32], float (&h)[32]) {
            if (args.act_kind == MOE_ACT_SWIGLU) {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float gv = __uint_as_float(g[j]);
                    const float uv = __uint_as_float(u[j]);
                    // silu(g) * u with the fast exponential and division (within
                    // the layer's tolerance; the division returns 0 where 1 + e^-g
                    // overflows, the limit of silu)
                    h[j] = __fdividef(gv * uv, 1.0f + __expf(-gv));
                }
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float gv = __uint_as_float(g[j]);
                    const float uv = __uint_as_float(u[j]);
                    // SiTU: sigmoid(g) * beta*tanh(g/beta) * lbeta*tanh(u/lbeta)
                    const float up = args.inv_lbeta != 0.0f ? args.lbeta * tanhf(uv * args.inv_lbeta) : uv;
                    h[j] = __fdividef(args.beta * tanhf(gv * args.inv_beta), 1.0f + __expf(-gv)) * up;
                }
            }
            };
            // FP8 requantisation of 32 tokens of h (this lane's row): the scale
            // byte of token cb*32 + lane (the amax over the warp's 32 rows, one
            // UE8M0 group of GEMM2's K) and the 32 codes, four tokens per word
            // (byte b of word m: token 4m + b)
            auto quantize8 = [&](float (&h)[32], uint32_t (&pq)[8], uint32_t &sfb) {
                float amx[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) amx[j] = fabsf(h[j]);
                const int e = scale_exponent<true>(warp_transpose_max(amx, lane));
                const float mult = exp2_neg(e);
                sfb = uint32_t(e + 127);
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    float v[4];
#pragma unroll
                    for (int b = 0; b < 4; ++b) v[b] = h[4 * m + b] * __shfl_sync(0xFFFFFFFFu, mult, 4 * m + b);
                    pq[m] = to_e4m3x4(v);
                }
            };
            // Stores of quantize8's results for column block cb: the scale byte,
            // then the codes.  Lanes 4G .. 4G+3 hold rows 4G .. 4G+3; a 4 x 4
            // byte transpose among them gives lane 4G + r the four row bytes of
            // token 4m + r, one 4-byte store per token and word.
            auto store8 = [&](const uint32_t (&pq)[8], uint32_t sfb, int cb) {
                const int tok = cb * 32 + lane;
                if (tok < ch.z)
                    args.out_sf[(int64_t(c) * n_tiles + it) * C::kActSf + act_sf_offset(tok, q)] = uint8_t(sfb);
                const int G = lane >> 2, r = lane & 3;
                const uint32_t sel = uint32_t(r) | (uint32_t(4 + r) << 4);
                uint8_t *qrow = args.out_q + (int64_t(it) * args.rows + ch.y + cb * 32) * kTileK + q * 32 + 4 * G;
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const uint32_t v0 = __shfl_sync(0xFFFFFFFFu, pq[m], 4 * G);
                    const uint32_t v1 = __shfl_sync(0xFFFFFFFFu, pq[m], 4 * G + 1);
                    const uint32_t v2 = __shfl_sync(0xFFFFFFFFu, pq[m], 4 * G + 2);
                    const uint32_t v3 = __shfl_sync(0xFFFFFFFFu, pq[m], 4 * G + 3);
                    const uint32_t w = __byte_perm(__byte_perm(v0, v1, sel), __byte_perm(v2, v3, sel), 0x5410);
                    const int t = 4 * m + r;
                    if (cb * 32 + t < ch.z) *reinterpret_cast<uint32_t *>(qrow + int64_t(t) * kTileK) = w;
                }
            };
            // NVFP4 requantisation of 32 tokens of h (this lane's row): groups of
            // 16 rows of h are the two half-warps; lane l gets the UE4M3 scale
            // codes of tokens cb*32 + l%16 (byte 0 of sc) and cb*32 + 16 + l%16
            // (byte 1), and its 32 E2M1 codes, eight per word (nibble j % 8 of
            // word j / 8: token j)
            auto quantize4 = [&](float (&h)[32], uint32_t (&cq)[4], uint32_t &sc) {
                float amx[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) amx[j] = fabsf(h[j]);
                float amA, amB;
                halfwarp_transpose_max(amx, lane, amA, amB);
                const uint32_t cA = nvfp4_scale_code(amA), cB = nvfp4_scale_code(amB);
                const float sA = e4m3_mag_value(cA), sB = e4m3_mag_value(cB);
                const float rA = __frcp_rn(sA), rB = __frcp_rn(sB);
                sc = cA | (cB << 8);
#pragma unroll
                for (int m = 0; m < 4; ++m) cq[m] = 0u;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int src = (lane & 16) | (j & 15);
                    const float sj = __shfl_sync(0xFFFFFFFFu, j < 16 ? sA : sB, src);
                    const float rj = __shfl_sync(0xFFFFFFFFu, j < 16 ? rA : rB, src);
                    cq[j >> 3] |= to_e2m1(nvfp4_quotient(h[j], sj, rj)) << (4 * (j & 7));
                }
            };
            // Stores of quantize4's results for column block cb: the two scale
            // bytes, then one byte per token from each even lane (its own code in
            // the low nibble, the next row's in the high one).  GEMM2 reads h in
            // 256-K blocks: this item's 128 rows are half `it % 2` of block it / 2,
            // and the warp's 32 rows are groups g4 = (q % 2) * 2 + half-warp of
            // image (it % 2) * 2 + q / 2.
            auto store4 = [&](const uint32_t (&cq)[4], uint32_t sc, int cb) {
                const int img = (it & 1) * 2 + (q >> 1), g4 = (q & 1) * 2 + (lane >> 4);
                uint8_t *sfo = args.out_sf + ((int64_t(c) * (n_tiles / 2) + it / 2) * kNvImages + img) * C::kActSf;
                const int tA = cb * 32 + (lane & 15), tB = tA + 16;
                if (tA < ch.z) sfo[act_sf_offset(tA, g4)] = uint8_t(sc & 0xFFu);
                if (tB < ch.z) sfo[act_sf_offset(tB, g4)] = uint8_t(sc >> 8);
                uint32_t pc[4];
#pragma unroll
                for (int m = 0; m < 4; ++m) pc[m] = __shfl_xor_sync(0xFFFFFFFFu, cq[m], 1);
                uint8_t *qbase = args.out_q + (int64_t(it >> 1) * args.rows + ch.y) * kTileK + (it & 1) * 64 +
                                 q * 16 + (lane >> 1);
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const uint32_t code = (cq[j >> 3] >> (4 * (j & 7))) & 0xFu;
                    const uint32_t partner = (pc[j >> 3] >> (4 * (j & 7))) & 0xFu;
                    if (!(lane & 1) && cb * 32 + j < ch.z)
                        qbase[int64_t(cb * 32 + j) * kTileK] = uint8_t(code | (partner << 4));
                }
            };
            // GEMM1 epilogue of 32 tokens: activation, scale, requantised h
            auto finish1 = [&](const uint32_t (&g)[32], const uint32_t (&u)[32], int cb) {
            float h[32];
            activate(g, u, h);
            if constexpr (kNv) {
                uint32_t cq[4], sc;
                quantize4(h, cq, sc);
                store4(cq, sc, cb);
            } else {
                uint32_t pq[8], sfb;
                quantize8(h, pq, sfb);
                store8(pq, sfb, cb);
            }
            };
            // GEMM2: 32 fp32 accumulator words (tokens) -> 16 words of bf16 pairs
            // (word m: token 2m in the low half, 2m + 1 in the high half)
            auto pack2 = [&](const uint32_t (&g)[32], uint32_t (&pk)[16]) {
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    const __nv_bfloat162 b2 =
                        __floats2bfloat162_rn(__uint_as_float(g[2 * m]), __uint_as_float(g[2 * m + 1]));
                    pk[m] = *reinterpret_cast<const uint32_t *>(&b2);
                }
            };
            // GEMM2 stores of 32 tokens of output tile 2 * it + a: bf16 Y rows
            auto store2 = [&](const uint32_t (&pk)[16], int a, int cb) {
                const int tile = 2 * it + a;
            __nv_bfloat16 *ybase = args.out_y + int64_t(ch.y + cb * 32) * args.out_ld + tile * kTileRows + q * 32;
            if constexpr (C::kStaged) {
                // two passes of 16 rows: stage [row][32 columns] bf16 (1 KB), then
                // 16-byte stores, four lanes per 64-byte row piece
                uint16_t *sb = reinterpret_cast<uint16_t *>(my_stage);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        sb[j * 32 + lane] = uint16_t(pk[hh * 8 + j / 2] >> (16 * (j & 1)));
                    __syncwarp();
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const int cidx = i * 32 + lane;  // row hh*16 + cidx / 4, columns (cidx % 4) * 8 ..
                        const int r = hh * 16 + (cidx >> 2);
                        if (cb * 32 + r < ch.z)
                            *reinterpret_cast<uint4 *>(ybase + int64_t(r) * args.out_ld + (cidx & 3) * 8) =
                                *reinterpret_cast<const uint4 *>(my_stage + cidx * 16);
                    }
                    __syncwarp();
                }
            } else {
                uint16_t *yb = reinterpret_cast<uint16_t *>(ybase);
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (cb * 32 + j < ch.z) yb[int64_t(j) * args.out_ld + lane] = uint16_t(pk[j / 2] >> (16 * (j & 1)));
            }
            };
            // GEMM2 epilogue of 32 tokens of output tile 2 * it + a (NVFP4, split
            // units): bf16 Y rows straight from the accumulator words
            auto finish2 = [&](const uint32_t (&g)[32], int a, int cb) {
                const int tile = 2 * it + a;
            __nv_bfloat16 *ybase = args.out_y + int64_t(ch.y + cb * 32) * args.out_ld + tile * kTileRows + q * 32;
            if constexpr (C::kStaged) {
                __nv_bfloat16 *sb = reinterpret_cast<__nv_bfloat16 *>(my_stage);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        sb[j * 32 + lane] = __float2bfloat16_rn(__uint_as_float(g[hh * 16 + j]));
                    __syncwarp();
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const int cidx = i * 32 + lane;
                        const int r = hh * 16 + (cidx >> 2);
                        if (cb * 32 + r < ch.z)
                            *reinterpret_cast<uint4 *>(ybase + int64_t(r) * args.out_ld + (cidx & 3) * 8) =
                                *reinterpret_cast<const uint4 *>(my_stage + cidx * 16);
                    }
                    __syncwarp();
                }
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (cb * 32 + j < ch.z)
                        ybase[int64_t(j) * args.out_ld + lane] = __float2bfloat16_rn(__uint_as_float(g[j]));
            }
            };
            // a split unit's partial: [tile][kN columns][128 rows] fp32
            float *part = is_unit ? args.part + size_t(P.unit) * kPartUnitFloats : nullptr;
            // (the chunk's real rows only: the item's last unit reads no others)
            auto put_part = [&](int a, int cb, const uint32_t (&v)[32]) {
                float *p = part + size_t(a * kN + cb * 32) * kTileRows + q * 32 + lane;
                const int nr = ch.z - cb * 32;
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (j < nr) p[j * kTileRows] = __uint_as_float(v[j]);
            };
            // Whole items: only the work that reads the accumulator runs while
            // the MMAs wait for it.  Each unit's results go to a few registers
            // (GEMM1: the requantised codes and scales; GEMM2: 16 words of bf16
            // pairs), the accumulator is released to the issuers, and then the
            // units' global stores run, overlapping the next item's MMAs.
            // (NVFP4's GEMM2 with 32-row chunks adds two K-split accumulators and
            // keeps the per-unit path: no registers to spare.)
            if (!is_unit && (!kNv || kGemm1 || !C::kSmall)) {
                if constexpr (kGemm1) {
                    // FP8: 8 words of codes + the scale byte per column block;
                    // NVFP4: 4 words of codes + the two scale codes
                    constexpr int kU = ((kN + 31) / 32 + kCbStep - 1) / kCbStep;
                    constexpr int kW = kNv ? 4 : 8;
                    uint32_t pq[kU][kW], sfb[kU];
#pragma unroll
                    for (int i = 0; i < kU; ++i) {
                        const int cb = half + i * kCbStep;
                        if (cb < ncb) {
                            uint32_t g[32], u[32];
                            float h[32];
                            load_gu(cb, g, u);
                            activate(g, u, h);
                            if constexpr (kNv)
                                quantize4(h, pq[i], sfb[i]);
                            else
                                quantize8(h, pq[i], sfb[i]);
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tmem_empty[buf]);
#pragma unroll
                    for (int i = 0; i < kU; ++i) {
                        const int cb = half + i * kCbStep;
                        if (cb < ncb) {
                            if constexpr (kNv)
                                store4(pq[i], sfb[i], cb);
                            else
                                store8(pq[i], sfb[i], cb);
                        }
                    }
                } else {
                    constexpr int kU = (kNumA * ((kN + 31) / 32) + kCbStep - 1) / kCbStep;
                    uint32_t pk[kU][16];
#pragma unroll
                    for (int i = 0; i < kU; ++i) {
                        const int u = half + i * kCbStep, a = u % kNumA, cb = u / kNumA;
                        if (cb < ncb && 2 * it + a < n_tiles) {
                            uint32_t g[32];
                            load_tile(a, cb, g);
                            pack2(g, pk[i]);
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tmem_empty[buf]);
#pragma unroll
                    for (int i = 0; i < kU; ++i) {
                        const int u = half + i * kCbStep, a = u % kNumA, cb = u / kNumA;
                        if (cb < ncb && 2 * it + a < n_tiles) store2(pk[i], a, cb);
                    }
                }
                continue;
            }
            if constexpr (kGemm1) {
                for (int cb = half; cb < ncb; cb += kCbStep) {
                    uint32_t g[32], u[32];
                    load_gu(cb, g, u);
                    if (is_unit) {
                        put_part(0, cb, g);
                        put_part(1, cb, u);
                    } else {
                        finish1(g, u, cb);
                    }
                }
            } else {
                // units (column block cb, tile a) = u / kNumA, u % kNumA: with two
                // warps per lane quarter each takes one tile's column blocks
#pragma unroll 1
                for (int u = half; u < kNumA * ncb; u += kCbStep) {
                    const int a = u % kNumA, cb = u / kNumA;
                    if (2 * it + a >= n_tiles) continue;
                    uint32_t g[32];
                    load_tile(a, cb, g);
                    if (is_unit)
                        put_part(a, cb, g);
                    else
                        finish2(g, a, cb);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tmem_empty[buf]);
            if (!is_unit) continue;
            // split unit: count it in; the item's last unit adds the partials of
            // units 0 .. split-1 in that order and finishes the item
            __threadfence();
            __syncwarp();
            if (lane == 0) mbar_arrive(epi_bar);
            if (warp == 2 && lane == 0) {
                int last = 0;
                if (mbar_wait(epi_bar, 0, abort_flag, err, 7)) {
                    __threadfence();
                    last = atomicAdd(args.split_cnt + P.unit / P.split, 1) == P.split - 1;
                    __threadfence();
                }
                *epi_last = last;
                mbar_arrive(epi_go);
            }
            if (!mbar_wait(epi_go, 0, abort_flag, err, 8)) break;
            if (!*epi_last) continue;
            const float *p0 = args.part + size_t(P.unit / P.split) * P.split * kPartUnitFloats;
            // tile a's sum over the units of column block cb, added in unit order;
            // rows past the chunk's end read as zero.  A block of at most 8 real
            // rows (decode) takes four units' loads per round.
            auto sum_part = [&](int a, int cb, uint32_t (&v)[32]) {
                const float *p = p0 + size_t(a * kN + cb * 32) * kTileRows + q * 32 + lane;
                const int nr = ch.z - cb * 32;
                if (nr <= 8) {
                    float s8[8];
#pragma unroll 1
                    for (int sp0 = 0; sp0 < P.split; sp0 += 4) {
                        float t[4][8];
#pragma unroll
                        for (int i = 0; i < 4; ++i)
#pragma unroll
                            for (int j = 0; j < 8; ++j)
                                t[i][j] = (sp0 + i < P.split && j < nr)
                                              ? __ldcg(p + size_t(sp0 + i) * kPartUnitFloats + j * kTileRows)
                                              : 0.0f;
#pragma unroll
                        for (int i = 0; i < 4; ++i)
#pragma unroll
                            for (int j = 0; j < 8; ++j)
                                if (sp0 + i == 0)
                                    s8[j] = t[i][j];
                                else if (sp0 + i < P.split)
                                    s8[j] += t[i][j];
                    }
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(j < 8 ? s8[j & 7] : 0.0f);
                    return;
                }
                float acc_v[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) acc_v[j] = j < nr ? __ldcg(p + j * kTileRows) : 0.0f;
                for (int sp = 1; sp < P.split; ++sp) {
                    p += kPartUnitFloats;
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (j < nr) acc_v[j] += __ldcg(p + j * kTileRows);
                }
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(acc_v[j]);
            };
            for (int cb = half; cb < ncb; cb += kCbStep) {
                if constexpr (kGemm1) {
                    uint32_t g[32], u[32];
                    sum_part(0, cb, g);
                    sum_part(1, cb, u);
                    finish1(g, u, cb);
                } else {
#pragma unroll 1
                    for (int a = 0; a < kNumA; ++a) {
                        if (2 * it + a >= n_tiles) break;
                        uint32_t g[32];
                        sum_part(a, cb, g);
                        finish2(g, a, cb);
                    }
                }
            }
        }
    }

    if (args.overlap_prev) pdl_wait();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
}

template <bool kGemm1, int kN, bool kNv>
static cudaError_t launch_gemm_t(const CUtensorMap &tmap_w, const CUtensorMap &tmap_wsf, const CUtensorMap &tmap_act,
                                 const CUtensorMap &tmap_act_full, const GemmArgs &args, int grid,
                                 cudaStream_t stream) {
    using C = GemmCfg<kGemm1, kN, kNv>;
    const cudaError_t e =
        set_max_dynamic_smem(reinterpret_cast<const void *>(moe_gemm_kernel<kGemm1, kN, kNv>), C::kSmemBytes);
    if (e != cudaSuccess) return e;
    return launch_pdl(moe_gemm_kernel<kGemm1, kN, kNv>, dim3(grid), dim3(C::kThreads), size_t(C::kSmemBytes), stream,
                      tmap_w, tmap_wsf, tmap_act, tmap_act_full, args);
}

template <bool kNv>
static int kblocks_per_stage(int chunk_rows) {
    return chunk_rows == kChunkRowsSmall ? GemmCfg<true, kChunkRowsSmall, kNv>::kKB
                                         : GemmCfg<true, kChunkRows, kNv>::kKB;
}

int gemm_kblocks_per_stage(int chunk_rows, bool nvfp4) {
    return nvfp4 ? kblocks_per_stage<true>(chunk_rows) : kblocks_per_stage<false>(chunk_rows);
}

int gemm_packets_per_stage(bool gemm1, int chunk_rows, bool nvfp4) {
    // every item owns two tiles; a stage moves both for each of its K blocks
    (void)gemm1;
    return 2 * gemm_kblocks_per_stage(chunk_rows, nvfp4);
}

template <bool kNv>
static cudaError_t launch_gemm_fmt(bool gemm1, bool small, const CUtensorMap &tmap_w, const CUtensorMap &tmap_wsf,
                                   const CUtensorMap &tmap_act, const CUtensorMap &tmap_act_full, const GemmArgs &a,
                                   int grid, cudaStream_t stream) {
    if (gemm1)
        return small ? launch_gemm_t<true, kChunkRowsSmall, kNv>(tmap_w, tmap_wsf, tmap_act, tmap_act_full, a, grid,
                                                                 stream)
                     : launch_gemm_t<true, kChunkRows, kNv>(tmap_w, tmap_wsf, tmap_act, tmap_act_full, a, grid, stream);
    return small ? launch_gemm_t<false, kChunkRowsSmall, kNv>(tmap_w, tmap_wsf, tmap_act, tmap_act_full, a, grid,
                                                              stream)
                 : launch_gemm_t<false, kChunkRows, kNv>(tmap_w, tmap_wsf, tmap_act, tmap_act_full, a, grid, stream);
}

cudaError_t launch_gemm(bool gemm1, const CUtensorMap &tmap_w, const CUtensorMap &tmap_wsf,
                        const CUtensorMap &tmap_act, const CUtensorMap &tmap_act_full, bool w_rowmajor,
                        uint8_t *ws, const WsLayout &L, int H, int I, int grid, cudaStream_t stream,
                        const moe_activation_t &act, bool nvfp4, bool side) {
    GemmArgs a{};
    a.w_rowmajor = w_rowmajor ? 1 : 0;
    a.w_rows_per_expert = gemm1 ? 2 * I : H;
    a.w_item_rows = gemm1 ? kTileRows : 2 * kTileRows;
    a.w_sf_x0 = w_rowmajor ? 0 : kPacketBody / 4;
    a.act_kind = act.kind;
    a.beta = act.beta;
    a.inv_beta = act.kind == MOE_ACT_SITU ? 1.0f / act.beta : 0.0f;
    a.lbeta = act.linear_beta;
    a.inv_lbeta = (act.kind == MOE_ACT_SITU && act.linear_beta > 0.0f) ? 1.0f / act.linear_beta : 0.0f;
    a.chunks = reinterpret_cast<const int4 *>(ws + (side ? L.off_chunks_s : L.off_chunks));
    a.hdr = reinterpret_cast<int *>(ws);
    a.chunks_word = side ? kHdrNumChunksSide : kHdrNumChunks;
    a.overlap_prev = side ? 1 : 0;
    a.part = reinterpret_cast<float *>(ws + L.off_part);
    a.split_cnt = a.hdr + (gemm1 ? kHdrSplitCnt1 : kHdrSplitCnt2);
    a.rows = int(L.Rp);
    const size_t xg_sf = side ? L.off_xg_sf_s : L.off_xg_sf, hq_sf = side ? L.off_hq_sf_s : L.off_hq_sf;
    if (gemm1) {
        a.act_sf = ws + xg_sf;
        a.out_q = ws + L.off_hq;
        a.out_sf = ws + hq_sf;
        a.K = H;
        a.n_tiles = I / kTileRows;
        a.n_items = I / kTileRows;
        a.out_ld = I;
    } else {
        a.act_sf = ws + hq_sf;
        a.out_y = reinterpret_cast<__nv_bfloat16 *>(ws + L.off_y);
        a.K = I;
        a.n_tiles = H / kTileRows;
        a.n_items = (H / kTileRows + 1) / 2;
        a.out_ld = H;
    }
    const bool small = side || L.chunk_rows == kChunkRowsSmall;
    return nvfp4 ? launch_gemm_fmt<true>(gemm1, small, tmap_w, tmap_wsf, tmap_act, tmap_act_full, a, grid, stream)
                 : launch_gemm_fmt<false>(gemm1, small, tmap_w, tmap_wsf, tmap_act, tmap_act_full, a, grid, stream);
}

}  // namespace moe
