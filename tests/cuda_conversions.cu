// Test infrastructure only: CUDA's own FP8 E4M3 and FP4 E2M1 conversions
// (cuda_fp8.h, cuda_fp4.h), exported through a C ABI so that the tests can
// pin the oracle's codebooks and round-to-nearest-even rule against a library
// routine: once on the host (the headers' host path) and once in a kernel on
// the GPU (the sm_100a conversion instructions).  Nothing in the layer's CUDA
// library or in the oracle uses this file.
//
// Every entry point returns 0 on success, else a cudaError_t value (device
// entries) or -1 for a bad argument.  Device entries take device pointers and
// a cudaStream_t (NULL = the legacy default stream) and return once the
// kernel is queued; the caller synchronises.
#include <cuda_bf16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__host__ __device__ float decode_e4m3(uint32_t code)
{
    __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)code, __NV_E4M3);
    return __half2float(__half(h));
}

__host__ __device__ float decode_e2m1(uint32_t code)
{
    __half_raw h = __nv_cvt_fp4_to_halfraw((__nv_fp4_storage_t)code, __NV_E2M1);
    return __half2float(__half(h));
}

__host__ __device__ uint8_t round_e4m3(float v)
{
    return (uint8_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}

__host__ __device__ uint8_t round_e2m1(float v)
{
    return (uint8_t)(__nv_cvt_float_to_fp4(v, __NV_E2M1, cudaRoundNearest) & 0xF);
}

// kind 0: decode E4M3 codes 0..n-1; 1: decode E2M1 codes 0..n-1
__global__ void decode_kernel(int kind, float *out, int n)
{
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
        out[i] = kind == 0 ? decode_e4m3((uint32_t)i) : decode_e2m1((uint32_t)i);
}

// kind 0: round to E4M3; 1: round to E2M1 (one code per byte, low nibble)
__global__ void round_kernel(int kind, const float *in, uint8_t *out, int n)
{
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
        out[i] = kind == 0 ? round_e4m3(in[i]) : round_e2m1(in[i]);
}

int grid_for(int n)
{
    int g = (n + 255) / 256;
    return g < 1 ? 1 : (g > 1184 ? 1184 : g);
}

}  // namespace

extern "C" {

// host path: out[0..255] / out[0..15] = the value of every code
int cvt_host_decode_e4m3(float *out)
{
    if (!out)
        return -1;
    for (uint32_t c = 0; c < 256; ++c)
        out[c] = decode_e4m3(c);
    return 0;
}

int cvt_host_decode_e2m1(float *out)
{
    if (!out)
        return -1;
    for (uint32_t c = 0; c < 16; ++c)
        out[c] = decode_e2m1(c);
    return 0;
}

// host path: out[i] = the code nearest in[i] (ties to even), i < n
int cvt_host_round_e4m3(const float *in, uint8_t *out, int n)
{
    if (n < 0 || (n > 0 && (!in || !out)))
        return -1;
    for (int i = 0; i < n; ++i)
        out[i] = round_e4m3(in[i]);
    return 0;
}

int cvt_host_round_e2m1(const float *in, uint8_t *out, int n)
{
    if (n < 0 || (n > 0 && (!in || !out)))
        return -1;
    for (int i = 0; i < n; ++i)
        out[i] = round_e2m1(in[i]);
    return 0;
}

// host path: out[i] = the UE8M0 byte of the smallest power of two >= |in[i]|
// (rounding toward +infinity, clipped to 2^-127 .. 2^127), i < n
int cvt_host_e8m0_ceil(const double *in, uint8_t *out, int n)
{
    if (n < 0 || (n > 0 && (!in || !out)))
        return -1;
    for (int i = 0; i < n; ++i)
        out[i] = (uint8_t)__nv_cvt_double_to_e8m0(in[i], __NV_SATFINITE, cudaRoundPosInf);
    return 0;
}

// host path: out[b] = the value of UE8M0 byte b, b < 256
int cvt_host_decode_e8m0(float *out)
{
    if (!out)
        return -1;
    for (uint32_t b = 0; b < 256; ++b)
        out[b] = __bfloat162float(__nv_bfloat16(__nv_cvt_e8m0_to_bf16raw((__nv_fp8_storage_t)b)));
    return 0;
}

// host path: out[i] = the bf16 bits of in[i] rounded to nearest even, i < n
int cvt_host_f32_to_bf16(const float *in, uint16_t *out, int n)
{
    if (n < 0 || (n > 0 && (!in || !out)))
        return -1;
    for (int i = 0; i < n; ++i) {
        const __nv_bfloat16 b = __float2bfloat16_rn(in[i]);
        out[i] = __nv_bfloat16_raw(b).x;
    }
    return 0;
}

// device path: the same on the GPU; out holds 256 / 16 floats
int cvt_dev_decode_e4m3(float *out, cudaStream_t stream)
{
    if (!out)
        return -1;
    decode_kernel<<<1, 256, 0, stream>>>(0, out, 256);
    return (int)cudaGetLastError();
}

int cvt_dev_decode_e2m1(float *out, cudaStream_t stream)
{
    if (!out)
        return -1;
    decode_kernel<<<1, 32, 0, stream>>>(1, out, 16);
    return (int)cudaGetLastError();
}

int cvt_dev_round_e4m3(const float *in, uint8_t *out, int n, cudaStream_t stream)
{
    if (n < 0 || (n > 0 && (!in || !out)))
        return -1;
    if (n == 0)
        return 0;
    round_kernel<<<grid_for(n), 256, 0, stream>>>(0, in, out, n);
    return (int)cudaGetLastError();
}

int cvt_dev_round_e2m1(const float *in, uint8_t *out, int n, cudaStream_t stream)
{
    if (n < 0 || (n > 0 && (!in || !out)))
        return -1;
    if (n == 0)
        return 0;
    round_kernel<<<grid_for(n), 256, 0, stream>>>(1, in, out, n);
    return (int)cudaGetLastError();
}

}  // extern "C"
