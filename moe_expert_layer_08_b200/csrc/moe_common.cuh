// moe_common.cuh -- sm_100a primitives shared by the kernels of the MoE layer:
// mbarriers, TMA (tiled and bulk, never multicast), tcgen05 (TMEM alloc, MMA,
// copies, loads), the UE8M0 scale rule and the device error word.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// ---------------------------------------------------------------- layout constants
constexpr int kTileRows = 128;        // weight rows per MMA (M) and per packet
constexpr int kTileK = 128;           // K elements per pipeline stage and per packet
constexpr int kChunkRows = 160;       // max routed rows (tokens) per work item (MMA N), large batches
constexpr int kChunkRowsSmall = 32;   // the same for small batches (decode)
constexpr int kBoxRows = 16;          // activation rows per TMA box
constexpr int kPacketBody = kTileRows * kTileK / 2;   // 8192 B of packed FP4
constexpr int kPacketSf = kTileRows * 4;              // 512 B of UE8M0 (4 groups x 128 rows)
constexpr int kPacketBytes = kPacketBody + kPacketSf; // 8704 B
constexpr int kSfBlockBytes = 128 * 4;                // 512 B scale image of 128 rows x 4 groups

// Bytes of the activation scale blocks of one (chunk, 128-K block): one
// 128-row image per 128 rows of the chunk.
__host__ __device__ constexpr int act_sf_bytes(int chunk_rows) { return (chunk_rows + 127) / 128 * kSfBlockBytes; }
// Offset of (row r < 256, group g) inside those blocks.
__host__ __device__ __forceinline__ int act_sf_offset(int r, int g);
constexpr int kMaxExperts = 1024;
constexpr int kMaxI = 8192;

// Device error word bits (workspace header word 0).
constexpr int kDevErrBadRouting = 1;
constexpr int kDevErrTimeout = 2;

// Workspace header (int32 words).
constexpr int kHdrError = 0;
constexpr int kHdrNumChunks = 1;
constexpr int kHdrDropped = 2;
constexpr int kHdrTimeoutWhere = 3;
constexpr int kHdrNumChunksSide = 4;  // chunks of the side list (large batches: lightly loaded experts)
constexpr int kProbeWhere = 99;       // kHdrTimeoutWhere value the bounded-wait probe records
// A per-expert chunk base with this bit set indexes the side list.
constexpr int kSideChunkBit = 1 << 30;
// Split-unit counters of the 32-row GEMMs (zeroed by routing on every forward):
// GEMM1 at words kHdrSplitCnt1.., GEMM2 at kHdrSplitCnt2.., one per leftover item.
constexpr int kMaxSplitUnits = 256;  // units per launch (leftover items x split)
constexpr int kHdrSplitWords = kMaxSplitUnits / 2;
constexpr int kHdrSplitCnt1 = 64;
constexpr int kHdrSplitCnt2 = kHdrSplitCnt1 + kHdrSplitWords;
constexpr int kHdrBytes = 2048;
static_assert(4 * (kHdrSplitCnt2 + kHdrSplitWords) <= kHdrBytes, "workspace header");
// fp32 partial accumulators of one split unit: two 128-row tiles x 32 tokens
constexpr int kPartUnitFloats = 2 * 32 * 128;

// Bounded waits: a device-side wait gives up after this many nanoseconds.
constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;

// Offset of byte (row r, group g in 0..3) inside a 512-byte scale block: the
// 32-lane x 16-byte image that tcgen05.cp .32x128b.warpx4 copies into TMEM,
// where lane r%32 holds rows r%32, r%32+32, r%32+64, r%32+96 in its 4 words.
__host__ __device__ __forceinline__ int sf_block_offset(int r, int g) {
    return (r & 31) * 16 + (r >> 5) * 4 + g;
}
__host__ __device__ __forceinline__ int act_sf_offset(int r, int g) {
    return (r >> 7) * kSfBlockBytes + sf_block_offset(r & 127, g);
}

// ---------------------------------------------------------------- UE8M0 scale rule
// e = smallest integer with amax <= qmax * 2^e, decided exactly from the bits
// of amax.  qmax is 448 = 1.75 * 2^8 (E4M3) or 6 = 1.5 * 2^2 (E2M1):
// writing amax = m * 2^E0 with m in [1, 2), e = E0 - p if m <= c else E0 - p + 1
// (c = 1.75, p = 8 or c = 1.5, p = 2).  amax = 0 gives e = 0.  Clamped to
// [-127, 127] so the scale byte e + 127 stays in [0, 254].
template <bool kFp8>
__device__ __forceinline__ int scale_exponent(float amax) {
    const uint32_t bits = __float_as_uint(amax);
    if (bits == 0u) return 0;
    int e0;
    uint32_t frac;
    if ((bits >> 23) != 0u) {
        e0 = int(bits >> 23) - 127;
        frac = bits & 0x7FFFFFu;
    } else {  // subnormal: normalise the mantissa
        const int msb = 31 - __clz(bits);
        e0 = msb - 149;
        frac = (bits << (23 - msb)) & 0x7FFFFFu;
    }
    const uint32_t c = kFp8 ? 0x600000u : 0x400000u;  // 0.75 or 0.5 of the mantissa
    int e = e0 - (kFp8 ? 8 : 2) + (frac > c ? 1 : 0);
    e = e < -127 ? -127 : e;
    e = e > 127 ? 127 : e;
    return e;
}

// 2^-e as fp32 (e in [-127, 126] gives a normal number).
__device__ __forceinline__ float exp2_neg(int e) {
    return __uint_as_float(uint32_t(127 - e) << 23);
}

// E4M3 code of v (already scaled, |v| <= 448), round to nearest even, sign bit
// from v (so values that round to zero keep their sign).
__device__ __forceinline__ uint32_t to_e4m3(float v) {
    const __nv_fp8_storage_t m = __nv_cvt_float_to_fp8(fabsf(v), __NV_SATFINITE, __NV_E4M3);
    return uint32_t(m) | ((__float_as_uint(v) >> 24) & 0x80u);
}

// The E4M3 codes of four scaled values, v[b] in byte b, two conversions per
// instruction; as in to_e4m3 the sign bit of every code is the sign bit of
// its value (a value that rounds to zero keeps its sign).
__device__ __forceinline__ uint32_t to_e4m3x4(const float (&v)[4]) {
    const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(v[0], v[1]), __NV_SATFINITE, __NV_E4M3);
    const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(v[2], v[3]), __NV_SATFINITE, __NV_E4M3);
    const uint32_t sign = ((__float_as_uint(v[0]) >> 24) & 0x80u) | ((__float_as_uint(v[1]) >> 16) & 0x8000u) |
                          ((__float_as_uint(v[2]) >> 8) & 0x800000u) | (__float_as_uint(v[3]) & 0x80000000u);
    return (lo | (hi << 16)) | sign;
}

// E2M1 code (4 bits) of v (|v| <= 6), round to nearest even, sign from v.
__device__ __forceinline__ uint32_t to_e2m1(float v) {
    const __nv_fp4_storage_t m = __nv_cvt_float_to_fp4(fabsf(v), __NV_E2M1, cudaRoundNearest);
    return (uint32_t(m) & 0xFu) | ((__float_as_uint(v) >> 28) & 0x8u);
}

// ---------------------------------------------------------------- NVFP4
// E2M1 values with one UE4M3 scale per 16 K elements.  A K block is 256
// elements (128 bytes of packed FP4, one 128-byte swizzled shared-memory row),
// and each of its four 64-K MMA steps takes one 512-byte scale image (4 groups
// of 16 for 128 rows, the same image layout as above).
constexpr int kNvTileK = 256;
constexpr int kNvImages = 4;                                  // scale images per 256-K block
constexpr int kNvPacketBody = kTileRows * kNvTileK / 2;       // 16384 B
constexpr int kNvPacketSf = kNvImages * kSfBlockBytes;        // 2048 B
constexpr int kNvPacketBytes = kNvPacketBody + kNvPacketSf;   // 18432 B

// Value of an E4M3 magnitude code c in [0, 126], exactly.
__device__ __forceinline__ float e4m3_mag_value(uint32_t c) {
    const uint32_t e = c >> 3, m = c & 7u;
    return e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : float(m) * (1.0f / 512.0f);
}

// NVFP4 scale code of a 16-element group: the smallest UE4M3 value s with
// 6 * s >= amax (6 * s is exact in fp32), found from a rounded estimate and
// exact comparisons; amax = 0 gives 1.0 (code 0x38); at most 0x7E (448).
__device__ __forceinline__ uint32_t nvfp4_scale_code(float amax) {
    if (!(amax > 0.0f)) return 0x38u;
    uint32_t c = uint32_t(__nv_cvt_float_to_fp8(amax * (1.0f / 6.0f), __NV_SATFINITE, __NV_E4M3)) & 0x7Fu;
    if (c == 0u) c = 1u;
    while (c < 0x7Eu && 6.0f * e4m3_mag_value(c) < amax) ++c;
    while (c > 1u && 6.0f * e4m3_mag_value(c - 1u) >= amax) --c;
    return c;
}

// h / s rounded to nearest (the fp32 quotient an E2M1 code is taken from),
// for an UE4M3 scale s > 0 and r = RN(1 / s), without a division per value:
// q0 = RN(h r), then one correction from the exact remainder h - q0 s (an
// FMA), q = RN(q0 + (h - q0 s) r) -- the reciprocal-based correction step of
// P. Markstein, "IA-64 and Elementary Functions" (2000), ch. 8.  An exhaustive
// GPU comparison with the IEEE division (all 126 nonzero UE4M3 magnitudes,
// every fp32 h with 2^-60 <= |h| < 2^101) found no difference.  Outside that
// range, and where |q0| >= 8, the last bits cannot change the E2M1 code:
// there q0 itself is used (|h / s| < 2^-51 rounds to a zero code with the sign
// of h), clamped to +-8 (which saturates to the largest code like any
// quotient above 6).
__device__ __forceinline__ float nvfp4_quotient(float h, float s, float r) {
    const float q0 = __fmul_rn(h, r);
    const float rem = __fmaf_rn(-q0, s, h);
    const float q = __fmaf_rn(rem, r, q0);
    const bool exact = fabsf(h) >= 0x1p-60f && fabsf(q0) < 8.0f;
    return exact ? q : fminf(fmaxf(q0, -8.0f), 8.0f);
}

// ---------------------------------------------------------------- misc
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_timer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0u;
}

// Bounded wait for the phase of `bar` with the given parity.  Gives up when
// another role has raised `abort` or after kWaitTimeoutNs, in which case it
// raises `abort`, records `where` and the timeout bit in the error word.
static __device__ __noinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort,
                                       int *err_word, int where,
                                       unsigned long long timeout_ns = kWaitTimeoutNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if (global_timer_ns() - t0 > timeout_ns) {
            *abort = 1;
            atomicOr(err_word + kHdrError, kDevErrTimeout);
            atomicExch(err_word + kHdrTimeoutWhere, where);
            return false;
        }
    }
}

// ---------------------------------------------------------------- programmatic dependent launch
// Block until the preceding kernel on the stream has completed and its memory
// is visible (no-op when the kernel was not launched as a dependent).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Allow the next kernel on the stream to be scheduled once every CTA of this
// grid has issued this (or exited).
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------- TMA (no multicast)
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1,
                                            uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1,
                                            int c2, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tma_load_4d(void *dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1,
                                            int c2, int c3, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5, %6}], [%2], %7;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "l"(policy)
        : "memory");
}

// Untiled bulk copy global -> shared (16-byte aligned addresses, size % 16 == 0).
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                          uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive once on `bar` when all tcgen05 operations issued so far by this thread complete.
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}
// Copy a 512-byte scale block (32 rows x 16 B in shared memory) to TMEM lanes
// 0..31 of 4 columns, replicated into all four 32-lane quarters.
__device__ __forceinline__ void tc_cp_sf(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
// D[M=128, N] (+)= (A * SFA) . (B * SFB)^T, block-scaled, fp32 accumulator in TMEM.
__device__ __forceinline__ void tc_mma_mxf8f6f4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// D[M=128, N] (+)= (A * SFA) . (B * SFB)^T with A and B both packed E2M1 and
// UE4M3 scales per 16 K (K = 64 per instruction; sfa / sfb address the
// 4-column scale image of this 64-K step).
__device__ __forceinline__ void tc_mma_nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// D[M=128, N] (+)= A . B^T with A and B both bf16 (K = 16 per instruction,
// 32 bytes of each operand row), fp32 accumulator in TMEM.
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 32 lanes x 32 columns of 32-bit words: thread l of the warp gets lane (base + l).
__device__ __forceinline__ void tmem_ld_32x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor, K-major, 128-byte swizzle: rows of 128 B,
// 8-row groups 1024 B apart (SBO), tile base 1024-byte aligned.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= uint64_t((saddr >> 4) & 0x3FFFu);
    d |= uint64_t(1) << 16;                 // LBO (unused for swizzled K-major)
    d |= uint64_t(1024 >> 4) << 32;         // SBO
    d |= uint64_t(1) << 46;                 // descriptor version (sm_100)
    d |= uint64_t(2) << 61;                 // SWIZZLE_128B
    return d;
}
// Descriptor of a 512-byte scale block for tcgen05.cp: no swizzle, 8-row x
// 16-byte core matrices 128 B apart.
__device__ __forceinline__ uint64_t smem_desc_sf(uint32_t saddr) {
    uint64_t d = 0;
    d |= uint64_t((saddr >> 4) & 0x3FFFu);
    d |= uint64_t(128 >> 4) << 32;
    d |= uint64_t(1) << 46;
    return d;
}
// Instruction descriptor of kind::f16 MMA: fp32 accumulator, A and B both
// bf16 (format 1), K-major, M = 128, N = n.
__device__ __forceinline__ uint32_t idesc_bf16(uint32_t n) {
    return (1u << 4)             // D format: F32
           | (1u << 7)           // A format: BF16
           | (1u << 10)          // B format: BF16
           | ((n >> 3) << 17)    // N / 8
           | ((128u >> 4) << 24);// M / 16
}
// Instruction descriptor of kind::mxf4nvf4 block-scaled MMA with 16-element
// scale vectors: A and B E2M1 (format 1), K-major, M = 128, N = n, UE4M3
// scales (scale format 0), dense K = 64.
__device__ __forceinline__ uint32_t idesc_nvf4(uint32_t n) {
    return (1u << 7)             // A format: E2M1
           | (1u << 10)          // B format: E2M1
           | ((n >> 3) << 17)    // N / 8
           | (0u << 23)          // scale format: UE4M3
           | ((128u >> 4) << 24);// M / 16
}
// Instruction descriptor of kind::mxf8f6f4 block-scaled MMA: A = E2M1 weights,
// B = E4M3 activations, both K-major, M = 128, N = n, UE8M0 scales, byte `id`
// of each 32-bit scale word (K step id of the 128-K stage).
__device__ __forceinline__ uint32_t idesc_mxf8f6f4(uint32_t n, uint32_t id) {
    return (id << 4)             // B scale factor id
           | (5u << 7)           // A format: E2M1
           | (0u << 10)          // B format: E4M3
           | ((n >> 3) << 17)    // N / 8
           | (1u << 23)          // scale format: UE8M0
           | ((128u >> 4) << 24) // M / 16
           | (id << 29);         // A scale factor id
}

}  // namespace moe
