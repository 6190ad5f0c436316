/*
 * moe.h -- C ABI of the B200 (sm_100a) FP8 x FP4 MoE expert layer.
 *
 * One MoE expert layer on one GPU: top-k routing to a per-expert token
 * permutation, grouped GEMM1 of FP8 E4M3 activations against FP4 E2M1 expert
 * weights (both with one UE8M0 scale per 32 elements along K), SwiGLU fused
 * with an FP8 E4M3 + UE8M0 requantisation, grouped GEMM2, and a top-k-weighted
 * combine back to bf16 tokens.  It restates, for a single GPU, the five-phase
 * "Mega MoE" pipeline of the pages "Mega moe fusion with symmetric memory"
 * (Procedure, step 5: dispatch, GEMM1, SwiGLU, GEMM2, combine) and MATE's
 * "Mega MoE" API page (API: get_symm_buffer_for_mega_moe,
 * transform_weights_for_mega_moe, fp8_fp8_mega_moe); the cross-rank dispatch
 * and combine become a local gather and a local weighted scatter.
 *
 * Conventions for every entry point:
 *  - All array pointers are DEVICE pointers (cudaMalloc / torch CUDA tensors)
 *    unless stated otherwise; arrays are dense, row-major, contiguous.
 *  - The caller owns every buffer; no entry point allocates device memory.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and the host is never synchronised, except by
 *    moe_check_device_error and moe_read_routing, which say so.
 *  - Arguments are validated on the host before any CUDA call.  A rejected
 *    call returns a non-zero moe_status_t and touches no memory.
 *  - FP4 E2M1 is packed two per byte, element 2c in the low nibble of byte c.
 *  - UE8M0 scale bytes b mean 2^(b-127) and are stored in K order: byte g of
 *    a row scales elements 32g .. 32g+31 of that row.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *moe_stream_t; /* same type as cudaStream_t */

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,        /* null / misaligned pointer, negative size */
    MOE_ERR_UNSUPPORTED_SHAPE = 2,  /* H or I not a multiple of 128, I > 8192, E > 1024, ... */
    MOE_ERR_WORKSPACE_TOO_SMALL = 3,
    MOE_ERR_CUDA = 4,               /* a CUDA runtime / driver call failed */
    MOE_ERR_BAD_ROUTING = 5,        /* device-detected expert id outside [0, E) */
    MOE_ERR_DEVICE_TIMEOUT = 6      /* a bounded device-side wait gave up */
} moe_status_t;

/* Number of events moe_forward records when given an event array. */
#define MOE_NUM_STAGE_EVENTS 5

/* Human-readable name of a status code (static string, never NULL). */
const char *moe_status_string(int status);

/* Library ABI version (increments on any signature change). */
int moe_abi_version(void);

/*
 * moe_quantize_fp8 -- per-row, per-32 FP8 E4M3 quantisation with UE8M0 scales
 * (the activation cast `per_token_cast_to_fp8(x, use_ue8m0=True, gran_k=32)`
 * of the DeepGEMM PR #416 review thread, test body).
 *   x      : bf16 [rows, cols], cols % 32 == 0, 16-byte aligned
 *   q      : u8   [rows, cols]      E4M3 codes (out)
 *   sf     : u8   [rows, cols/32]   UE8M0 bytes (out)
 * Per group of 32: e = smallest integer with amax <= 448 * 2^e (amax = 0 gives
 * e = 0), scale byte e+127 clamped to [0, 254]; code = round-to-nearest-even
 * of v * 2^-e, sign bit = sign bit of v.  Same rule as the layer's SwiGLU
 * requantisation.
 */
moe_status_t moe_quantize_fp8(const void *x, int64_t rows, int64_t cols,
                              void *q, void *sf, moe_stream_t stream);

/*
 * moe_quantize_fp4 -- per-row, per-32 FP4 E2M1 quantisation with UE8M0 scales
 * (the weight cast `_cast_weights_to_fp4` of the same test body), same rule
 * with format maximum 6.
 *   w      : bf16 [rows, cols], cols % 32 == 0, 16-byte aligned
 *   q      : u8   [rows, cols/2]    packed E2M1 (out)
 *   sf     : u8   [rows, cols/32]   UE8M0 bytes (out)
 */
moe_status_t moe_quantize_fp4(const void *w, int64_t rows, int64_t cols,
                              void *q, void *sf, moe_stream_t stream);

/*
 * moe_transformed_weight_bytes -- sizes of the two tile-major weight buffers
 * that moe_transform_weights writes for E experts (host-only, no CUDA call):
 * 8704 bytes per packet (128 x 128 FP4 body + 512 scale bytes), 2*(I/128)*(H/128)
 * packets per expert for L1 and 2*ceil(H/256)*(I/128) for L2.
 */
moe_status_t moe_transformed_weight_bytes(int E, int H, int I,
                                          size_t *l1_bytes, size_t *l2_bytes);

/*
 * moe_transform_weights -- model-load-time layout transform
 * (`transform_weights_for_mega_moe(l1, l2, tile_pack=True)`: MATE "Mega MoE"
 * API; DeepGEMM PR #394 "cluster-paired FP4 weight packets", Summary and
 * Motivation).  Packs each expert's logical FP4 weights and their UE8M0
 * scales into packets of one 128-row x 128-K tile followed by the 512 scale
 * bytes that tile consumes, so body and scales share one allocation and one
 * access stream.  Packet order: expert -> intermediate tile i -> K tile ->
 * (gate tile i, up tile i) for L1; expert -> output tile pair p -> K tile ->
 * (tile 2p, tile 2p+1) for L2, so the two tiles one GEMM work item multiplies
 * are adjacent for every K tile (an odd H/128 gets one zero-filled padding
 * tile per expert).
 *   l1    : u8 [E, 2I, H/2]   rows 0..I-1 gate, I..2I-1 up     (in)
 *   l1_sf : u8 [E, 2I, H/32]                                   (in)
 *   l2    : u8 [E, H, I/2]                                     (in)
 *   l2_sf : u8 [E, H, I/32]                                    (in)
 *   l1_t, l2_t : outputs of moe_transformed_weight_bytes size, 256-byte aligned
 * H % 128 == 0, I % 128 == 0, I <= 8192.  To transform one expert at a time,
 * call with E = 1 and pointers offset to that expert: the packets of expert e
 * start at e * (l1_bytes / E) and e * (l2_bytes / E).
 */
moe_status_t moe_transform_weights(const void *l1, const void *l1_sf,
                                   const void *l2, const void *l2_sf,
                                   int E, int H, int I,
                                   void *l1_t, void *l2_t, moe_stream_t stream);

/*
 * moe_workspace_bytes -- device workspace moe_forward needs for up to T_max
 * tokens (host-only).  Holds the routing metadata (counts, offsets,
 * permutation and inverse, tile list), the gathered FP8 activations, the FP8
 * SwiGLU output with its scales and the bf16 GEMM2 rows: the runtime workspace
 * of MATE's "Mega MoE" page (Typical Flow), sized for the worst case.
 */
moe_status_t moe_workspace_bytes(int T_max, int E, int k, int H, int I, size_t *bytes);

/*
 * moe_forward_kernel_launches -- how many kernels one moe_forward or
 * moe_forward_act call with these sizes enqueues (host-only; no counterpart on
 * the pages: it lets a caller that counts launches, such as a benchmark or a
 * graph builder, know the layer's launch structure).  Routing takes two
 * kernels when T * k <= 1024 (one block does histogram, scan and placement,
 * then the gather) and five otherwise (histogram, per-expert scan, metadata,
 * placement, gather); GEMM1, GEMM2 and the combine add three.  When
 * T * k > 8 * E (160-row chunks) GEMM1 and GEMM2 run a second time, as the
 * 32-row kernels over the experts with at most 32 routed rows (two more).
 * T = 0 enqueues nothing.  Returns MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED_SHAPE for sizes
 * moe_forward would reject.
 */
moe_status_t moe_forward_kernel_launches(int T, int E, int k, int H, int I, int *launches);

/*
 * moe_forward -- one MoE expert layer (`fp8_fp4_mega_moe(y, l1, l2, buffer)`;
 * the five phases of "Mega moe fusion with symmetric memory", Procedure step 5,
 * on one GPU).
 *   x_fp8    : u8  [T, H]      E4M3 activations, 16-byte aligned
 *   x_sf     : u8  [T, H/32]   UE8M0 activation scales, 4-byte aligned
 *   topk_idx : i64 [T, k]      expert ids; an id outside [0, E) is dropped
 *                              (contributes nothing) and reported by
 *                              moe_check_device_error as MOE_ERR_BAD_ROUTING;
 *                              a repeated id counts as separate routed rows
 *   topk_w   : f32 [T, k]      combine weights
 *   l1_t, l2_t : buffers written by moe_transform_weights
 *   out_bf16 : bf16 [T, H]     out[t] = bf16_rne(sum_j topk_w[t,j] * Y(t,j)),
 *                              fully overwritten, 16-byte aligned
 *   workspace: >= moe_workspace_bytes(T, E, k, H, I) bytes, 256-byte aligned;
 *              its contents after the call are the routing metadata of this
 *              call (moe_read_routing) and scratch
 *   expert_stats : nullable i32 [E]; when given, expert_stats[e] += rows routed
 *              to e (the `cumulative_local_expert_recv_stats` of the API page)
 *   stage_events : nullable array of MOE_NUM_STAGE_EVENTS cudaEvent_t; when
 *              given, recorded on `stream` before routing, before GEMM1,
 *              before GEMM2, before the combine and after the combine
 * Computes per routed row r = (t, j, e): C1 = x[t] . L1[e]^T (fp32),
 * h = silu(C1[:, :I]) * C1[:, I:], h -> FP8 E4M3 + UE8M0 per 32 (the
 * moe_quantize_fp8 rule), Y = h . L2[e]^T (fp32, stored bf16), then the
 * weighted combine in ascending j.  T = 0 is a no-op.  The call is
 * asynchronous and performs no host synchronisation.
 */
moe_status_t moe_forward(const void *x_fp8, const void *x_sf,
                         const int64_t *topk_idx, const float *topk_w,
                         const void *l1_t, const void *l2_t, void *out_bf16,
                         int T, int E, int k, int H, int I,
                         void *workspace, size_t ws_bytes,
                         int32_t *expert_stats, void *const *stage_events,
                         moe_stream_t stream);

/*
 * Activation between GEMM1 and the FP8 requantisation (MATE "Mega MoE" API,
 * section Activations: "swiglu" by default, "situ" with a required positive
 * coefficient and an optional positive linear coefficient).
 *   MOE_ACT_SWIGLU: h = silu(gate) * up
 *   MOE_ACT_SITU:   h = sigmoid(gate) * beta*tanh(gate/beta)
 *                       * linear_beta*tanh(up/linear_beta)   (formula of the
 *                   DeepGEMM PR #416 test body); linear_beta = 0 means absent,
 *                   and then the up factor is `up` itself.
 */
typedef enum { MOE_ACT_SWIGLU = 0, MOE_ACT_SITU = 1 } moe_activation_kind_t;
typedef struct {
    int kind;           /* moe_activation_kind_t */
    float beta;         /* SiTU: > 0 and finite */
    float linear_beta;  /* SiTU: 0 (absent) or > 0 and finite */
} moe_activation_t;

/*
 * moe_forward_act -- moe_forward with a chosen activation.  `activation` is a
 * HOST pointer (read during the call; NULL = SwiGLU).  Everything else is as
 * for moe_forward; an invalid kind or coefficient returns MOE_ERR_INVALID_ARG
 * before any CUDA call.
 */
moe_status_t moe_forward_act(const void *x_fp8, const void *x_sf,
                             const int64_t *topk_idx, const float *topk_w,
                             const void *l1_t, const void *l2_t, void *out_bf16,
                             int T, int E, int k, int H, int I,
                             void *workspace, size_t ws_bytes,
                             int32_t *expert_stats, void *const *stage_events,
                             const moe_activation_t *activation, moe_stream_t stream);

/*
 * Weight layouts (DeepGEMM PR #394, Summary and API: the packet layout is an
 * option of the model-load transform; "row-major" weights keep their natural
 * layout).
 *   MOE_LAYOUT_PACKETS   l1 / l2 are the buffers of moe_transform_weights
 *                        (body and scales of each tile in one packet);
 *                        l1_sf / l2_sf must be NULL.
 *   MOE_LAYOUT_ROW_MAJOR l1 / l2 are the FP4 weights as moe_quantize_fp4 wrote
 *                        them (l1 [E, 2I, H/2], rows 0..I-1 gate; l2 [E, H, I/2]),
 *                        256-byte aligned, read in place; l1_sf / l2_sf are the
 *                        scale blocks of moe_transform_scales.
 * Both layouts feed the tensor cores the same bytes, so the layer's output is
 * bitwise identical between them.
 */
typedef enum { MOE_LAYOUT_PACKETS = 0, MOE_LAYOUT_ROW_MAJOR = 1 } moe_layout_t;
typedef struct {
    int layout;        /* moe_layout_t */
    const void *l1, *l1_sf;
    const void *l2, *l2_sf;
} moe_weights_t;

/*
 * moe_transformed_scale_bytes -- sizes of the separate scale arrays of the
 * row-major layout (host-only): 512 bytes per 128 x 128 weight tile, in the
 * packet order of moe_transform_weights (L1: E * (I/128) * (H/128) * 2 blocks;
 * L2: E * ceil(H/256) * 2 * (I/128) blocks, an odd H/128 padded with zero
 * blocks).
 */
moe_status_t moe_transformed_scale_bytes(int E, int H, int I, size_t *l1_sf_bytes, size_t *l2_sf_bytes);

/*
 * moe_transform_scales -- the scale half of moe_transform_weights: writes each
 * tile's 512-byte scale block (the image tcgen05.cp copies into TMEM, byte
 * (r % 32) * 16 + (r / 32) * 4 + g for tile row r, K group g) into l1_sf_t /
 * l2_sf_t (256-byte aligned, sizes from moe_transformed_scale_bytes) and
 * leaves the FP4 bodies where they are.  l1_sf [E, 2I, H/32], l2_sf [E, H,
 * I/32] as moe_quantize_fp4 wrote them.  Same validation as
 * moe_transform_weights.
 */
moe_status_t moe_transform_scales(const void *l1_sf, const void *l2_sf, int E, int H, int I,
                                  void *l1_sf_t, void *l2_sf_t, moe_stream_t stream);

/*
 * moe_forward_weights -- moe_forward_act with the weights given by layout
 * (`weights` is a HOST pointer read during the call).  An unknown layout, a
 * missing or misaligned weight pointer, or l1_sf / l2_sf given with packets
 * returns MOE_ERR_INVALID_ARG before any CUDA call.  No counterpart on the
 * pages beyond the layout option itself: it lets one runtime serve both
 * layouts for their A/B comparison.
 */
moe_status_t moe_forward_weights(const void *x_fp8, const void *x_sf,
                                 const int64_t *topk_idx, const float *topk_w,
                                 const moe_weights_t *weights, void *out_bf16,
                                 int T, int E, int k, int H, int I,
                                 void *workspace, size_t ws_bytes,
                                 int32_t *expert_stats, void *const *stage_events,
                                 const moe_activation_t *activation, moe_stream_t stream);

/*
 * NVFP4 variant ("NVFP4 Mega MoE Kernel -- Mojo Rewrite" README: Key
 * operations, NVFP4 specifics): activations, weights and the intermediate h
 * are all FP4 E2M1 with one UE4M3 scale per 16 consecutive K elements, and the
 * GEMMs run tcgen05.mma.kind::mxf4nvf4.block_scale.scale_vec::4X.  Scale
 * rule (the pages give none): s = the smallest UE4M3 value with 6*s >= amax
 * (amax = 0 gives 1), code = E2M1 round-to-nearest-even of the fp32 quotient
 * v / s.  H % 256 == 0 and I % 256 == 0.
 */

/*
 * moe_quantize_nvfp4 -- bf16 [rows, cols] (16-byte aligned) -> packed E2M1 q
 * [rows, cols/2] (even element in the low nibble, 8-byte aligned) and UE4M3
 * sf [rows, cols/16].  cols % 16 == 0.
 */
moe_status_t moe_quantize_nvfp4(const void *x, int64_t rows, int64_t cols,
                                void *q, void *sf, moe_stream_t stream);

/*
 * moe_transformed_weight_bytes_nvfp4 -- packet buffer sizes of the NVFP4
 * weights (host-only): packets of 18432 bytes = 128 rows x 256 K of packed
 * E2M1 (16384 B) + four 512-byte UE4M3 scale images (one per 64 K), in the
 * same order as moe_transform_weights' packets with 256-K tiles.
 */
moe_status_t moe_transformed_weight_bytes_nvfp4(int E, int H, int I,
                                                size_t *l1_bytes, size_t *l2_bytes);

/*
 * moe_transform_weights_nvfp4 -- l1 [E, 2I, H/2], l1_sf [E, 2I, H/16],
 * l2 [E, H, I/2], l2_sf [E, H, I/16] as moe_quantize_nvfp4 wrote them ->
 * packets in l1_t / l2_t (256-byte aligned).  Validation as
 * moe_transform_weights.
 */
moe_status_t moe_transform_weights_nvfp4(const void *l1, const void *l1_sf,
                                         const void *l2, const void *l2_sf,
                                         int E, int H, int I,
                                         void *l1_t, void *l2_t, moe_stream_t stream);

/*
 * moe_forward_nvfp4 -- the layer in NVFP4: x_fp4 [T, H/2] packed E2M1
 * (16-byte aligned), x_sf [T, H/16] UE4M3 (4-byte aligned), l1_t / l2_t from
 * moe_transform_weights_nvfp4; everything else as moe_forward_act (the same
 * workspace size serves both formats).
 */
moe_status_t moe_forward_nvfp4(const void *x_fp4, const void *x_sf,
                               const int64_t *topk_idx, const float *topk_w,
                               const void *l1_t, const void *l2_t, void *out_bf16,
                               int T, int E, int k, int H, int I,
                               void *workspace, size_t ws_bytes,
                               int32_t *expert_stats, void *const *stage_events,
                               const moe_activation_t *activation, moe_stream_t stream);

/*
 * moe_read_routing -- copies the routing metadata of the last moe_forward that
 * used `workspace` with these (T, E, k, H, I) into HOST arrays (test and
 * inspection hook; synchronises `stream`).  Any output may be NULL.
 *   count  : i32 [E]     rows routed to each expert
 *   offset : i32 [E+1]   exclusive scan of count
 *   perm   : i32 [T*k]   perm[r] = t*k+j of routed row r, rows of one expert
 *                        in ascending t*k+j; entries >= offset[E] unused
 *   inv    : i32 [T*k]   inv[t*k+j] = r, or -1 for a dropped slot
 */
moe_status_t moe_read_routing(const void *workspace, int T, int E, int k, int H, int I,
                              int32_t *count, int32_t *offset, int32_t *perm,
                              int32_t *inv, moe_stream_t stream);

/*
 * moe_check_device_error -- synchronises `stream`, then reads the device error
 * word of the last moe_forward on `workspace`: MOE_OK, MOE_ERR_BAD_ROUTING
 * (an expert id was out of range) or MOE_ERR_DEVICE_TIMEOUT (a bounded wait
 * inside a kernel gave up; that call's output is undefined).
 */
moe_status_t moe_check_device_error(const void *workspace, moe_stream_t stream);

/*
 * moe_forward_static -- moe_forward without a caller-provided workspace, for
 * callers that cannot allocate device memory.  The pages have no counterpart
 * of this entry point; it exists for this library's users.
 *
 * Who cannot allocate: code that runs while a CUDA graph is being captured
 * (cudaMalloc is not a stream operation and is not allowed there), serving
 * runtimes that reserve all device memory for their own pools at start-up and
 * forbid allocation on the request path, and plug-ins called from inside
 * another framework's operator that cannot reach that framework's allocator
 * and must not call cudaMalloc, which can synchronise the device.
 *
 * Arguments and results are those of moe_forward, minus the workspace: the
 * caller still passes (and owns) every input and the output.  The layer's
 * scratch is one file-scope device array of MOE_STATIC_WORKSPACE_BYTES inside
 * this library, which every GPU that loads the library holds until the
 * process exits.  This entry point allocates nothing: no cudaMalloc, no
 * cudaFree, no allocating library routine.
 *  - The first call on a device looks up the array's device address on that
 *    device (cudaGetSymbolAddress); make that first call before any stream
 *    capture on that device.
 *  - A (T, E, k, H, I) whose moe_workspace_bytes exceeds
 *    MOE_STATIC_WORKSPACE_BYTES is rejected with MOE_ERR_WORKSPACE_TOO_SMALL
 *    before any device work (decode-sized batches fit: T = 128 tokens at
 *    E = 384, top-6, H = 7168, I = 3072 needs 57.9 MiB).
 *  - All calls on a device share the one array, which keeps the last call's
 *    contents; nothing in it needs to start at zero.  Calls that overlap on
 *    the GPU (different streams, or threads without ordering between their
 *    streams) race on it and give undefined results: issue them in order on
 *    one stream.
 *  - Out-of-range expert ids are dropped as in moe_forward.  The device
 *    error word of the last call lives in the shared array; read it with
 *    moe_check_device_error_static on that device.
 */
#define MOE_STATIC_WORKSPACE_BYTES (64u * 1024u * 1024u)

moe_status_t moe_forward_static(const void *x_fp8, const void *x_sf,
                                const int64_t *topk_idx, const float *topk_w,
                                const void *l1_t, const void *l2_t, void *out_bf16,
                                int T, int E, int k, int H, int I,
                                int32_t *expert_stats, void *const *stage_events,
                                moe_stream_t stream);

/*
 * moe_check_device_error_static -- moe_check_device_error for the fixed array
 * of moe_forward_static on CUDA device `device`: synchronises `stream`, then
 * returns the status the last moe_forward_static on that device left in the
 * array's error word (MOE_OK, MOE_ERR_BAD_ROUTING or MOE_ERR_DEVICE_TIMEOUT).
 * The first kernel of every moe_forward_static rewrites the word, so the
 * result belongs to the last call enqueued before `stream` was synchronised
 * (call it on the stream the forward ran on).  MOE_ERR_INVALID_ARG for a
 * device index outside [0, 64); allocates nothing.
 */
moe_status_t moe_check_device_error_static(int device, moe_stream_t stream);

/*
 * moe_probe_wait_timeout -- diagnostic (no counterpart on the pages): runs one
 * thread through the library's bounded device-side wait on a barrier that
 * nothing completes, with a limit of timeout_us microseconds (1 .. 1e6)
 * instead of the kernels' 2 s.  The wait gives up and records the timeout in
 * the workspace's error word, after which moe_check_device_error(workspace)
 * returns MOE_ERR_DEVICE_TIMEOUT and the context stays usable.  Enqueues a
 * 2 KiB memset of the workspace header and one kernel; workspace 256-byte
 * aligned, ws_bytes >= 2048.  Exercises the failure path without a fault.
 */
moe_status_t moe_probe_wait_timeout(void *workspace, size_t ws_bytes, unsigned timeout_us,
                                    moe_stream_t stream);

/*
 * BF16 shared expert (DeepGEMM PR #416, "BF16 shared expert" test body: an
 * optional dense expert that runs on every token beside the routed experts,
 * with bf16 input, weights and its own bf16 output).  With x [T, SH],
 * L1 [2 SI, SH] (rows 0..SI-1 gate, SI..2 SI-1 up) and L2 [SH, SI]:
 *   gate, up = bf16_rne(x . L1^T);  h = bf16_rne(act(gate, up));
 *   y = bf16_rne(h . L2^T)
 * with fp32 accumulation on the tensor cores (tcgen05 kind::f16) and act
 * SwiGLU or SiTU (moe_activation_t, as for the routed layer).
 *
 * moe_shared_workspace_bytes -- bytes of device workspace moe_shared_forward
 *   needs for up to T_max tokens (a 2 KiB header with the device error word,
 *   then h [T, SI] bf16, then the fp32 partial sums of the K split that
 *   token counts with fewer work items than SMs use: 8 MiB up to 64 tokens,
 *   16 MiB up to 128, 20 MiB above; the size never falls as T_max grows).
 *   MOE_ERR_UNSUPPORTED_SHAPE unless SH and SI are multiples of 128.
 *
 * moe_shared_forward -- y for T tokens.  All pointers are device pointers on
 *   one device, row-major and contiguous: x_bf16 [T, SH], l1_bf16 [2 SI, SH],
 *   l2_bf16 [SH, SI], out_bf16 [T, SH] (fully overwritten), all 16-byte
 *   aligned; workspace 256-byte aligned, ws_bytes >= moe_shared_workspace_bytes
 *   (T, SH, SI) (else MOE_ERR_WORKSPACE_TOO_SMALL).  activation NULL means
 *   SwiGLU.  The caller owns every buffer; the call allocates nothing,
 *   enqueues two kernels on `stream` (nothing else, so the first can start
 *   under the tail of the preceding kernel), and does not synchronise.
 *   T = 0 enqueues nothing.  The workspace must be zero-filled (e.g. by
 *   cudaMemsetAsync) before its first use by this entry point, and again
 *   after any other use of the same memory; every call leaves it ready for
 *   the next one, a call that timed out included.  Argument errors
 *   (MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED_SHAPE) are returned before any
 *   CUDA call; a device-side wait that times out is reported by
 *   moe_check_device_error(workspace) as MOE_ERR_DEVICE_TIMEOUT (the word
 *   holds the status of the last call).
 */
moe_status_t moe_shared_workspace_bytes(int T_max, int SH, int SI, size_t *bytes);
moe_status_t moe_shared_forward(const void *x_bf16, const void *l1_bf16, const void *l2_bf16,
                                void *out_bf16, int T, int SH, int SI,
                                const moe_activation_t *activation, void *workspace, size_t ws_bytes,
                                moe_stream_t stream);

/*
 * Expert parallelism: the per-rank ends of the dispatch and combine phases of
 * "Mega moe fusion with symmetric memory" (Procedure, step 5, phases 1 and 5;
 * MATE "Mega MoE" API page, Typical Flow), with the exchange between ranks
 * left to the caller (an all-to-all-v, e.g. NCCL through torch.distributed).
 * Rank r of R holds experts [r E/R, (r+1) E/R) (E % R == 0).  One step:
 *   1. moe_ep_dispatch on every rank: its T tokens' routed rows, grouped by
 *      destination rank, and the per-rank row counts;
 *   2. exchange the counts, then the rows (x, scales, local expert ids);
 *   3. on every rank, moe_forward over the received rows with E/R experts,
 *      k = 1, topk_idx = the received local ids and topk_w = 1, which yields
 *      each received row's bf16 expert output Y unchanged;
 *   4. send those outputs back (the reverse all-to-all-v);
 *   5. moe_ep_combine on every rank: out = the top-k-weighted sum, as
 *      moe_forward's own combine forms it.
 * With R = 1 (no exchange) the result equals moe_forward's bit for bit.
 *
 * moe_ep_workspace_bytes -- bytes of the dispatch workspace for up to T_max
 *   tokens (the routing metadata only: a 2 KiB header with the device error
 *   word, counts, offsets, permutation and its inverse, ...).
 *
 * moe_ep_dispatch -- routing plus the send buffers, in routing order (by
 *   expert, then by slot t*k+j; a dropped slot, id outside [0, E), has no row
 *   and is reported by moe_check_device_error(workspace)):
 *   x_fp8 u8 [T, H] (16-byte aligned), x_sf u8 [T, H/32] (4-byte aligned),
 *   topk_idx i64 [T, k] as for moe_forward;
 *   send_x u8 [T k, H] (16-byte aligned), send_sf u8 [T k, H/32] (4-byte
 *   aligned), send_eid i64 [T k] (the row's expert id minus its rank's first
 *   expert): the first n = sum(send_counts) rows are written;
 *   send_counts i64 [ranks] (rows for each destination rank, device memory).
 *   workspace 256-byte aligned, ws_bytes >= moe_ep_workspace_bytes(T, E, k, H);
 *   it must stay untouched until the matching moe_ep_combine.  H must be a
 *   multiple of 128.  T = 0 only zeroes send_counts.  Asynchronous on `stream`.
 *
 * moe_ep_combine -- out_bf16 [T, H] (16-byte aligned, fully overwritten) =
 *   bf16_rne(sum_{j ascending} topk_w[t, j] * y_bf16[inv[t k + j]]), fp32 sum,
 *   no atomics; y_bf16 [n, H] holds the rows returned for the dispatched rows,
 *   in send order; inv is the inverse permutation the dispatch with the same
 *   T, E, k, H left in the workspace.  T = 0 enqueues nothing.
 *
 * moe_ep_route -- step 1 without the copies, for moe_ep_dispatch_peers: the
 *   routing into the workspace and send_counts (i64 [ranks], device); the
 *   same arguments and rules as moe_ep_dispatch.
 *
 * moe_ep_dispatch_peers -- steps 1 and 2 for rows: after moe_ep_route with the
 *   same T, E, k, H, ranks and workspace, and once every rank's counts are
 *   known, writes each routed row (x_fp8 row, its UE8M0 scales, its local
 *   expert id) straight into the receive buffers of the rank that holds its
 *   expert, mapped into this rank's address space (CUDA IPC or symmetric
 *   memory over NVLink).  peer_x / peer_sf / peer_eid: device arrays [ranks]
 *   of device pointers to rank d's u8 [rows, H] (16-byte aligned), u8
 *   [rows, H/32] (4-byte aligned) and i64 [rows] receive buffers (an entry
 *   may be NULL only for a rank this rank sends nothing to); recv_base: i64
 *   [ranks] device, the row at which this rank's block starts in rank d's
 *   buffers (the sum of what ranks 0..r-1 send to d).  The rows land as the
 *   all-to-all of moe_ep_dispatch's send buffers would place them (source
 *   rank major, then send order).  The caller orders rank d's step 3 after
 *   every rank's call (e.g. a stream-ordered barrier).
 *
 * moe_ep_combine_peers -- steps 4 and 5 in one kernel, for ranks whose
 *   expert-layer outputs are mapped into this rank's address space (CUDA IPC
 *   or symmetric memory over NVLink): each returned row is read where rank d
 *   left it instead of being sent back first.  peer_y: device array [ranks]
 *   of device pointers, rank d's bf16 [rows, H] output of step 3 (16-byte
 *   aligned; an entry may be NULL only for a rank that holds none of this
 *   rank's rows); recv_base: i64 [ranks] device, the row at which this rank's
 *   block starts in rank d's received rows (the sum of what ranks 0..r-1
 *   sent to d); topk_idx and topk_w as for the dispatch.  The result equals
 *   moe_ep_combine's for the same rows bit for bit.  The caller orders the
 *   call after every rank's step 3 (e.g. a stream-ordered barrier) and keeps
 *   the peers' outputs until it completes.
 *
 * Argument errors (MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED_SHAPE /
 * MOE_ERR_WORKSPACE_TOO_SMALL) are returned before any CUDA call; a launch
 * failure is MOE_ERR_CUDA.  The caller owns every buffer.
 */
moe_status_t moe_ep_workspace_bytes(int T_max, int E, int k, int H, size_t *bytes);
moe_status_t moe_ep_dispatch(const void *x_fp8, const void *x_sf, const int64_t *topk_idx, int T, int E, int k,
                             int H, int ranks, void *workspace, size_t ws_bytes, void *send_x, void *send_sf,
                             int64_t *send_eid, int64_t *send_counts, moe_stream_t stream);
moe_status_t moe_ep_combine(const void *y_bf16, const float *topk_w, int T, int E, int k, int H,
                            const void *workspace, size_t ws_bytes, void *out_bf16, moe_stream_t stream);
moe_status_t moe_ep_route(const int64_t *topk_idx, int T, int E, int k, int H, int ranks, void *workspace,
                          size_t ws_bytes, int64_t *send_counts, moe_stream_t stream);
moe_status_t moe_ep_dispatch_peers(const void *x_fp8, const void *x_sf, const int64_t *topk_idx, int T, int E, int k,
                                   int H, int ranks, const void *workspace, size_t ws_bytes,
                                   void *const *peer_x, void *const *peer_sf, int64_t *const *peer_eid,
                                   const int64_t *recv_base, moe_stream_t stream);
moe_status_t moe_ep_combine_peers(const void *const *peer_y, const int64_t *recv_base, const int64_t *topk_idx,
                                  const float *topk_w, int T, int E, int k, int H, int ranks, const void *workspace,
                                  size_t ws_bytes, void *out_bf16, moe_stream_t stream);

/*
 * Peer buffers for the two entry points above (no counterpart on the pages,
 * which leave the symmetric-memory set-up to the serving system): CUDA IPC
 * over one process per GPU.
 *
 * moe_ipc_handle -- the IPC handle (MOE_IPC_HANDLE_BYTES bytes, written to
 *   `handle`) of the device allocation that holds device pointer `ptr`, and
 *   ptr's byte offset inside that allocation (`offset`), to be sent to the
 *   other ranks.  `ptr` may point anywhere inside an allocation (framework
 *   allocators sub-allocate).  Host-side only; enqueues nothing.
 * moe_ipc_open -- maps another process's allocation, given its handle, into
 *   this process on CUDA device `device` (peer access enabled as needed);
 *   `*base` receives the mapped base, to which the sender's offset is added.
 *   A process cannot open a handle of its own allocations (use the pointer).
 * moe_ipc_close -- unmaps a base returned by moe_ipc_open.  The mapping must
 *   outlive every kernel that reads or writes through it.
 * Errors: MOE_ERR_INVALID_ARG for null arguments or a negative device;
 * MOE_ERR_CUDA when CUDA refuses (the CUDA error is cleared).
 */
#define MOE_IPC_HANDLE_BYTES 64
moe_status_t moe_ipc_handle(const void *ptr, void *handle, size_t *offset);
moe_status_t moe_ipc_open(const void *handle, int device, void **base);
moe_status_t moe_ipc_close(void *base);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
