// combine.cu -- the top-k-weighted combine back to token order (phase 5 of
// "Mega moe fusion with symmetric memory", Procedure step 5, on one GPU: a
// local gather through the inverse permutation instead of cross-rank stores).
// out[t] = bf16_rne(sum_{j ascending} topk_w[t, j] * Y[inv[t*k + j]]), fp32
// sum, no atomics, so the result is deterministic.
#include "ep_internal.h"
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

constexpr int kCombineThreads = 128;
constexpr int kCombineCols = kCombineThreads * 8;  // 8 bf16 (16 bytes) per thread
constexpr int kCombineBatch = 8;                   // top-k up to this many: loads issued together

__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const __nv_bfloat16 *__restrict__ y,
                                                                  const int *__restrict__ inv,
                                                                  const float *__restrict__ topk_w, int k, int H,
                                                                  int col_blocks, int T,
                                                                  __nv_bfloat16 *__restrict__ out) {
    pdl_wait();
    pdl_trigger();
    // blocks stride over (token, 1024-column block) tasks
    for (int64_t task = blockIdx.x; task < int64_t(T) * col_blocks; task += gridDim.x) {
        const int64_t t = task / col_blocks;
        const int col = int(task % col_blocks) * kCombineCols + threadIdx.x * 8;
        if (col >= H) continue;
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
        auto add = [&](const uint4 &v, float wv) {
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                acc[2 * i] += wv * __uint_as_float(u[i] << 16);
                acc[2 * i + 1] += wv * __uint_as_float(u[i] & 0xFFFF0000u);
            }
        };
        if (k <= kCombineBatch) {
            // all of the token's row indices, then all row loads in flight at once;
            // the sum still runs over j ascending
            int r[kCombineBatch];
            float wv[kCombineBatch];
            uint4 v[kCombineBatch];
#pragma unroll
            for (int j = 0; j < kCombineBatch; ++j) {
                r[j] = j < k ? __ldcg(inv + t * k + j) : -1;
                wv[j] = j < k ? __ldg(topk_w + t * k + j) : 0.0f;
            }
#pragma unroll
            for (int j = 0; j < kCombineBatch; ++j)
                if (r[j] >= 0) v[j] = __ldcg(reinterpret_cast<const uint4 *>(y + int64_t(r[j]) * H + col));
#pragma unroll
            for (int j = 0; j < kCombineBatch; ++j)
                if (r[j] >= 0) add(v[j], wv[j]);  // r < 0: dropped slot
        } else {
            for (int j = 0; j < k; ++j) {
                const int r = __ldcg(inv + t * k + j);
                if (r < 0) continue;  // dropped slot
                add(__ldcg(reinterpret_cast<const uint4 *>(y + int64_t(r) * H + col)), __ldg(topk_w + t * k + j));
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

cudaError_t launch_combine_rows(const void *y, const int *inv, const float *topk_w, int T, int k, int H, void *out,
                                cudaStream_t stream) {
    const int col_blocks = (H + kCombineCols - 1) / kCombineCols;
    // at most 16 blocks (2048 threads) per SM, each looping over tasks: fewer,
    // longer-lived blocks than one per task keep more loads in flight
    const int64_t tasks = int64_t(T) * col_blocks, cap = int64_t(num_sms()) * 16;
    const int64_t grid = tasks < cap ? tasks : cap;
    return launch_pdl(combine_kernel, dim3(unsigned(grid)), dim3(kCombineThreads), 0, stream,
                      static_cast<const __nv_bfloat16 *>(y), inv, topk_w, k, H, col_blocks, T,
                      static_cast<__nv_bfloat16 *>(out));
}

cudaError_t launch_combine(const uint8_t *ws, const WsLayout &L, const float *topk_w, int T, int k, int H,
                           void *out, cudaStream_t stream) {
    return launch_combine_rows(ws + L.off_y, reinterpret_cast<const int *>(ws + L.off_inv), topk_w, T, k, H, out,
                               stream);
}

}  // namespace moe
