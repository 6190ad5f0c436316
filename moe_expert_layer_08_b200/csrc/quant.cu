// quant.cu -- the per-32 UE8M0 quantisers (activation cast to FP8 E4M3 and
// weight cast to FP4 E2M1, the casts of the DeepGEMM PR #416 review thread's
// test body), the NVFP4 quantiser (E2M1 with UE4M3 per 16, the NVFP4 Mega MoE
// README's format), and the model-load weight transforms into tile packets
// (DeepGEMM PR #394, "cluster-paired FP4 weight packets": body and scale words
// of one tile stored together, in the order the GEMM reads them).
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

// One thread per group of 32 consecutive elements of a row: 64 bytes of bf16
// in, 32 bytes (FP8) or 16 bytes (FP4) of codes and one scale byte out.
template <bool kFp8>
__global__ void __launch_bounds__(256) quantize_kernel(const __nv_bfloat16 *__restrict__ x, int64_t rows,
                                                       int64_t cols, uint8_t *__restrict__ q,
                                                       uint8_t *__restrict__ sf) {
    const int64_t gpr = cols / 32;
    const int64_t g = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (g >= rows * gpr) return;
    const uint4 *src = reinterpret_cast<const uint4 *>(x + g * 32);
    float v[32];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 w = __ldg(src + i);
        const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v[i * 8 + j * 2] = __uint_as_float(u[j] << 16);
            v[i * 8 + j * 2 + 1] = __uint_as_float(u[j] & 0xFFFF0000u);
        }
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const int e = scale_exponent<kFp8>(amax);
    const float m = exp2_neg(e);
    sf[g] = uint8_t(e + 127);
    if (kFp8) {
        uint32_t w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            w[i] = to_e4m3(v[4 * i] * m) | (to_e4m3(v[4 * i + 1] * m) << 8) | (to_e4m3(v[4 * i + 2] * m) << 16) |
                   (to_e4m3(v[4 * i + 3] * m) << 24);
        uint4 *dst = reinterpret_cast<uint4 *>(q + g * 32);
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    } else {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t acc = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) acc |= to_e2m1(v[8 * i + j] * m) << (4 * j);
            w[i] = acc;
        }
        *reinterpret_cast<uint4 *>(q + g * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

cudaError_t launch_quantize(const void *x, int64_t rows, int64_t cols, void *q, void *sf, bool fp8,
                            cudaStream_t stream) {
    const int64_t groups = rows * (cols / 32);
    if (groups == 0) return cudaSuccess;
    const int64_t blocks = (groups + 255) / 256;
    if (fp8)
        quantize_kernel<true><<<unsigned(blocks), 256, 0, stream>>>(
            static_cast<const __nv_bfloat16 *>(x), rows, cols, static_cast<uint8_t *>(q), static_cast<uint8_t *>(sf));
    else
        quantize_kernel<false><<<unsigned(blocks), 256, 0, stream>>>(
            static_cast<const __nv_bfloat16 *>(x), rows, cols, static_cast<uint8_t *>(q), static_cast<uint8_t *>(sf));
    return cudaGetLastError();
}

// One 128-thread block per packet (grid-stride): thread r copies the 64 bytes
// of row r of the tile and writes that row's 4 scale bytes into the packet's
// 512-byte scale block.  Packet p = ((e * groups + grp) * KB + kb) * 2 + slot
// holds K columns kb * 128 + [0, 128) of source rows
//   L1 (halves):  slot * half_rows + grp * 128 + [0, 128)   (slot 0 gate, 1 up)
//   L2 (pairs):   (2 * grp + slot) * 128 + [0, 128)         (two adjacent tiles)
// so the two tiles one GEMM item multiplies are adjacent for every K tile.  A
// pair slot past the last tile (odd tile count) is zero-filled padding.
// Without bodies (the row-major layout) output block p is packet p's 512-byte
// scale block alone, in the same order.
__global__ void __launch_bounds__(128) transform_kernel(const uint8_t *__restrict__ w, const uint8_t *__restrict__ w_sf,
                                                        int rows_per_expert, int K, int groups, bool pairs,
                                                        int half_rows, int64_t num_packets, uint8_t *__restrict__ out,
                                                        bool with_body) {
    const int KB = K / kTileK;
    const int r = threadIdx.x;
    for (int64_t p = blockIdx.x; p < num_packets; p += gridDim.x) {
        int64_t q = p;
        const int slot = int(q % 2);
        q /= 2;
        const int kb = int(q % KB);
        q /= KB;
        const int grp = int(q % groups);
        const int64_t e = q / groups;
        const int64_t row_in_expert =
            pairs ? int64_t(2 * grp + slot) * kTileRows + r : int64_t(slot) * half_rows + int64_t(grp) * kTileRows + r;
        uint8_t *pkt = with_body ? out + p * kPacketBytes : nullptr;
        uint4 *dst = with_body ? reinterpret_cast<uint4 *>(pkt + r * (kTileK / 2)) : nullptr;
        uint32_t *dsf = reinterpret_cast<uint32_t *>((with_body ? pkt + kPacketBody : out + p * kPacketSf) +
                                                     sf_block_offset(r, 0));
        if (row_in_expert >= rows_per_expert) {  // padding slot
            if (with_body) {
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[i] = make_uint4(0, 0, 0, 0);
            }
            *dsf = 0;
            continue;
        }
        const int64_t src_row = e * rows_per_expert + row_in_expert;
        if (with_body) {
            const uint4 *src = reinterpret_cast<const uint4 *>(w + src_row * (K / 2) + kb * (kTileK / 2));
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = __ldg(src + i);
        }
        *dsf = __ldg(reinterpret_cast<const uint32_t *>(w_sf + src_row * (K / 32) + kb * 4));
    }
}

// NVFP4: one thread per group of 16 consecutive elements of a row: 32 bytes of
// bf16 in, 8 bytes of packed E2M1 codes (even element in the low nibble) and
// one UE4M3 scale byte out.  Code = E2M1 round-to-nearest-even of the fp32
// quotient v / s, sign kept.
__global__ void __launch_bounds__(256) quantize_nvfp4_kernel(const __nv_bfloat16 *__restrict__ x, int64_t rows,
                                                             int64_t cols, uint8_t *__restrict__ q,
                                                             uint8_t *__restrict__ sf) {
    const int64_t gpr = cols / 16;
    const int64_t g = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (g >= rows * gpr) return;
    const uint4 *src = reinterpret_cast<const uint4 *>(x + g * 16);
    float v[16];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const uint4 w = __ldg(src + i);
        const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v[i * 8 + j * 2] = __uint_as_float(u[j] << 16);
            v[i * 8 + j * 2 + 1] = __uint_as_float(u[j] & 0xFFFF0000u);
        }
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const uint32_t c = nvfp4_scale_code(amax);
    const float s = e4m3_mag_value(c);
    sf[g] = uint8_t(c);
    uint32_t w[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        uint32_t acc = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) acc |= to_e2m1(__fdiv_rn(v[8 * i + j], s)) << (4 * j);
        w[i] = acc;
    }
    *reinterpret_cast<uint2 *>(q + g * 8) = make_uint2(w[0], w[1]);
}

cudaError_t launch_quantize_nvfp4(const void *x, int64_t rows, int64_t cols, void *q, void *sf, cudaStream_t stream) {
    const int64_t groups = rows * (cols / 16);
    if (groups == 0) return cudaSuccess;
    quantize_nvfp4_kernel<<<unsigned((groups + 255) / 256), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(x), rows, cols, static_cast<uint8_t *>(q), static_cast<uint8_t *>(sf));
    return cudaGetLastError();
}

// NVFP4 packets: the same enumeration as the FP8 x FP4 packets with 256-K
// tiles; a packet is 128 rows x 128 bytes of packed E2M1 (16384 B) followed by
// four 512-byte scale images (image s: groups 4s .. 4s+3, i.e. K elements
// 64s .. 64s+63 of the tile).  One 128-thread block per packet, thread r =
// tile row r.
__global__ void __launch_bounds__(128) transform_nv_kernel(const uint8_t *__restrict__ w,
                                                           const uint8_t *__restrict__ w_sf, int rows_per_expert, int K,
                                                           int groups, bool pairs, int half_rows, int64_t num_packets,
                                                           uint8_t *__restrict__ out) {
    const int KB = K / kNvTileK;
    const int r = threadIdx.x;
    for (int64_t p = blockIdx.x; p < num_packets; p += gridDim.x) {
        int64_t q = p;
        const int slot = int(q % 2);
        q /= 2;
        const int kb = int(q % KB);
        q /= KB;
        const int grp = int(q % groups);
        const int64_t e = q / groups;
        const int64_t row_in_expert =
            pairs ? int64_t(2 * grp + slot) * kTileRows + r : int64_t(slot) * half_rows + int64_t(grp) * kTileRows + r;
        uint8_t *pkt = out + p * kNvPacketBytes;
        uint4 *dst = reinterpret_cast<uint4 *>(pkt + r * (kNvTileK / 2));
        if (row_in_expert >= rows_per_expert) {  // padding slot
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int s = 0; s < kNvImages; ++s)
                *reinterpret_cast<uint32_t *>(pkt + kNvPacketBody + s * kSfBlockBytes + sf_block_offset(r, 0)) = 0;
            continue;
        }
        const int64_t src_row = e * rows_per_expert + row_in_expert;
        const uint4 *src = reinterpret_cast<const uint4 *>(w + src_row * (K / 2) + kb * (kNvTileK / 2));
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[i] = __ldg(src + i);
        const uint32_t *ssrc = reinterpret_cast<const uint32_t *>(w_sf + src_row * (K / 16) + kb * 16);
#pragma unroll
        for (int s = 0; s < kNvImages; ++s)
            *reinterpret_cast<uint32_t *>(pkt + kNvPacketBody + s * kSfBlockBytes + sf_block_offset(r, 0)) =
                __ldg(ssrc + s);
    }
}

cudaError_t launch_transform_nv(const void *w, const void *w_sf, int E, int rows_per_expert, int K, int groups,
                                bool pairs, int half_rows, void *out, cudaStream_t stream) {
    const int64_t num_packets = int64_t(E) * groups * (K / kNvTileK) * 2;
    if (num_packets == 0) return cudaSuccess;
    const int64_t grid = num_packets < 65536 ? num_packets : 65536;
    transform_nv_kernel<<<unsigned(grid), 128, 0, stream>>>(static_cast<const uint8_t *>(w),
                                                            static_cast<const uint8_t *>(w_sf), rows_per_expert, K,
                                                            groups, pairs, half_rows, num_packets,
                                                            static_cast<uint8_t *>(out));
    return cudaGetLastError();
}

cudaError_t launch_transform(const void *w, const void *w_sf, int E, int rows_per_expert, int K, int groups,
                             bool pairs, int half_rows, void *out, bool with_body, cudaStream_t stream) {
    const int64_t num_packets = int64_t(E) * groups * (K / kTileK) * 2;
    if (num_packets == 0) return cudaSuccess;
    const int64_t grid = num_packets < 65536 ? num_packets : 65536;
    transform_kernel<<<unsigned(grid), 128, 0, stream>>>(static_cast<const uint8_t *>(w),
                                                         static_cast<const uint8_t *>(w_sf), rows_per_expert, K,
                                                         groups, pairs, half_rows, num_packets,
                                                         static_cast<uint8_t *>(out), with_body);
    return cudaGetLastError();
}

}  // namespace moe
