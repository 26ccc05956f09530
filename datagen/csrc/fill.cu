// fill.cu - GPU implementation of the seeded input generator defined in
// datagen/__init__.py (counter-based SplitMix64, Irwin-Hall sum of twelve
// 16-bit uniforms). It fills multi-GB K/V caches in place; the host
// implementation regenerates any element bit for bit. Input generation only:
// no arithmetic of the LSA method lives here.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

__host__ __device__ __forceinline__ uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

__device__ __forceinline__ float normal_at(uint64_t key, uint64_t idx) {
    int32_t acc = 0;
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        const uint64_t w = mix64(key + (3ull * idx + (uint64_t)(j + 1)) * kGamma);
        acc += (int32_t)(w & 0xFFFFu) + (int32_t)((w >> 16) & 0xFFFFu) +
               (int32_t)((w >> 32) & 0xFFFFu) + (int32_t)(w >> 48);
    }
    return (float)(acc - 393210) * (1.0f / 65536.0f);
}

__device__ __forceinline__ uint16_t bf16_rne(float x) {
    uint32_t u = __float_as_uint(x);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

template <bool BF16>
__global__ void k_fill(void* dst, uint64_t count, uint64_t key, uint64_t first) {
    const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += stride) {
        const float x = normal_at(key, first + i);
        if constexpr (BF16) static_cast<uint16_t*>(dst)[i] = bf16_rne(x);
        else static_cast<float*>(dst)[i] = x;
    }
}

}  // namespace

extern "C" __attribute__((visibility("default")))
int dg_fill_normal(void* dst, int bf16, uint64_t count, uint32_t seed, uint32_t tensor_id,
                   uint64_t first_index, void* stream) {
    if (dst == nullptr) return 1;
    if (count == 0) return 0;
    const uint64_t key = mix64(((uint64_t)seed << 32) | tensor_id);
    int sms = 148, dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    uint64_t blocks = (count + 255) / 256;
    if (blocks > (uint64_t)sms * 32) blocks = (uint64_t)sms * 32;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (bf16) k_fill<true><<<(unsigned)blocks, 256, 0, st>>>(dst, count, key, first_index);
    else k_fill<false><<<(unsigned)blocks, 256, 0, st>>>(dst, count, key, first_index);
    return cudaGetLastError() == cudaSuccess ? 0 : 2;
}
