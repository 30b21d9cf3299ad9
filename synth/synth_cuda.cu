// Seeded synthetic inputs, device side.
//
// The CUDA twin of synth.c: the same SplitMix64 counter stream, the same
// Irwin-Hall(12) normal and the same bf16 rounding, so that weight banks of
// several GB can be generated in place in device memory with the exact bits
// the host generator gives.  It holds none of the mixture-of-experts
// arithmetic and is used only to make inputs.
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace {

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

__device__ __forceinline__ uint64_t sm64(uint64_t s, uint64_t i) {
    return mix64(s + (i + 1ULL) * 0x9E3779B97F4A7C15ULL);
}

__device__ __forceinline__ float irwin_hall12(uint64_t key, uint64_t j) {
    int32_t s = 0;
#pragma unroll
    for (int a = 0; a < 3; ++a) {
        uint64_t w = sm64(key, 3 * j + a);
#pragma unroll
        for (int q = 0; q < 4; ++q) s += (int32_t)((w >> (16 * q)) & 0xFFFFu);
    }
    int32_t n = s + 6 - 6 * 65536;
    return __fmul_rn(__int2float_rn(n), 1.0f / 65536.0f);
}

__global__ void normal_bf16_kernel(uint64_t key, uint64_t offset, uint64_t n, float sigma,
                                   __nv_bfloat16* __restrict__ out) {
    uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        float v = __fmul_rn(irwin_hall12(key, offset + i), sigma);
        out[i] = __float2bfloat16_rn(v);
    }
}

__global__ void normal_f32_kernel(uint64_t key, uint64_t offset, uint64_t n, float sigma,
                                  float* __restrict__ out) {
    uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
        out[i] = __fmul_rn(irwin_hall12(key, offset + i), sigma);
}

int grid_for(uint64_t n) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    uint64_t want = (n + 255) / 256;
    uint64_t cap = (uint64_t)sms * 8;
    return (int)(want < cap ? (want ? want : 1) : cap);
}

}  // namespace

extern "C" int synth_normal_bf16_cuda(uint64_t key, uint64_t offset, uint64_t n, float sigma,
                                      void* out, void* stream) {
    if (n == 0) return 0;
    normal_bf16_kernel<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(
        key, offset, n, sigma, (__nv_bfloat16*)out);
    return (int)cudaGetLastError();
}

extern "C" int synth_normal_f32_cuda(uint64_t key, uint64_t offset, uint64_t n, float sigma,
                                     void* out, void* stream) {
    if (n == 0) return 0;
    normal_f32_kernel<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(
        key, offset, n, sigma, (float*)out);
    return (int)cudaGetLastError();
}
