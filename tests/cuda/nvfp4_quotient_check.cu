// Test probe (built by tests/test_gpu_nvfp4_quotient.py): compares the NVFP4
// requantisation's division-free quotient (nvfp4_quotient in moe_common.cuh)
// with CUDA's correctly rounded division, bit for bit where the helper
// promises the exact quotient and by E2M1 code everywhere, for every nonzero
// UE4M3 scale magnitude and every finite fp32 h (or every `step`-th bit
// pattern).
#include <cstdint>
#include <cuda_runtime.h>

#include "moe_common.cuh"

using namespace moe;

__global__ void quotient_check(uint32_t code, uint32_t step, unsigned long long *bad_bits,
                               unsigned long long *bad_code) {
    const float s = e4m3_mag_value(code);
    const float r = __frcp_rn(s);
    const uint64_t stride = uint64_t(gridDim.x) * blockDim.x * step;
    for (uint64_t i = (uint64_t(blockIdx.x) * blockDim.x + threadIdx.x) * step; i < (1ull << 32); i += stride) {
        const uint32_t hb = uint32_t(i);
        const uint32_t ex = (hb >> 23) & 0xFFu;
        if (ex == 0xFFu) continue;  // inf / NaN
        const float h = __uint_as_float(hb);
        const float q_ref = __fdiv_rn(h, s);
        const float q = nvfp4_quotient(h, s, r);
        const bool exact_range = fabsf(h) >= 0x1p-60f && fabsf(__fmul_rn(h, r)) < 8.0f;
        if (exact_range && __float_as_uint(q) != __float_as_uint(q_ref)) atomicAdd(bad_bits, 1ull);
        // the codes of the IEEE quotient itself where it is finite (E2M1 saturates above 6)
        const float q_cmp = isfinite(q_ref) ? q_ref : fminf(fmaxf(q_ref, -8.0f), 8.0f);
        if (to_e2m1(q) != to_e2m1(q_cmp)) atomicAdd(bad_code, 1ull);
    }
}

// Mismatch counts over scale codes 1..126: [0] quotient bits, [1] E2M1 codes.
extern "C" int run_quotient_check(uint32_t step, unsigned long long *host_counts) {
    unsigned long long *d = nullptr;
    if (cudaMalloc(&d, 16) != cudaSuccess) return 1;
    cudaMemset(d, 0, 16);
    for (uint32_t c = 1; c <= 126; ++c) quotient_check<<<148 * 8, 256>>>(c, step, d, d + 1);
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemcpy(host_counts, d, 16, cudaMemcpyDeviceToHost);
    cudaFree(d);
    return e == cudaSuccess ? 0 : 2;
}
