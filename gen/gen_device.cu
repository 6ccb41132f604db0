// Seeded synthetic inputs, device side: the same counter-based generator as
// gen_host.c (SplitMix64 output function, Irwin-Hall(12) normals with an
// exact fp32 result, nearest-even rounding to bf16), written again for the
// GPU so large workloads are produced in place.  Test/bench infrastructure
// only; it holds none of the method's arithmetic.
#include <cstdint>
#include <cuda_runtime.h>

namespace {
constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ULL;

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
    z ^= z >> 30; z *= 0xBF58476D1CE4E5B9ULL;
    z ^= z >> 27; z *= 0x94D049BB133111EBULL;
    z ^= z >> 31;
    return z;
}

__device__ __forceinline__ float normal_at(uint64_t key, uint64_t i) {
    int32_t s = 0;
#pragma unroll
    for (int w = 0; w < 3; ++w) {
        uint64_t r = mix64(key + kGamma * (3 * i + (uint64_t)w + 1));
        s += (int32_t)(r & 0xFFFF) + (int32_t)((r >> 16) & 0xFFFF)
           + (int32_t)((r >> 32) & 0xFFFF) + (int32_t)(r >> 48);
    }
    return __int2float_rn(2 * s - 12 * 65535) * (1.0f / 131072.0f);
}

__device__ __forceinline__ uint16_t f32_to_bf16_rne(float x) {
    uint32_t u = __float_as_uint(x);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

__global__ void normal_bf16_kernel(uint64_t key, uint64_t offset, int64_t n, uint16_t* out) {
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < n;
         j += (int64_t)gridDim.x * blockDim.x)
        out[j] = f32_to_bf16_rne(normal_at(key, offset + (uint64_t)j));
}

__global__ void normal_f32_kernel(uint64_t key, uint64_t offset, int64_t n, float* out) {
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < n;
         j += (int64_t)gridDim.x * blockDim.x)
        out[j] = normal_at(key, offset + (uint64_t)j);
}

int grid_for(int64_t n) {
    int64_t g = (n + 255) / 256;
    if (g > 148 * 64) g = 148 * 64;
    if (g < 1) g = 1;
    return (int)g;
}
}  // namespace

extern "C" int gen_dev_normal_bf16(uint64_t key, uint64_t offset, int64_t n, void* out, void* stream) {
    if (n <= 0) return 0;
    normal_bf16_kernel<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(key, offset, n, (uint16_t*)out);
    return (int)cudaGetLastError();
}

extern "C" int gen_dev_normal_f32(uint64_t key, uint64_t offset, int64_t n, void* out, void* stream) {
    if (n <= 0) return 0;
    normal_f32_kernel<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(key, offset, n, (float*)out);
    return (int)cudaGetLastError();
}
