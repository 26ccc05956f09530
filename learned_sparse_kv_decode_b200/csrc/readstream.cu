// readstream.cu - a plain DRAM read stream, the ceiling the read-only hot path is compared with.
//
// Not a step of the method: a measurement utility. The split attention reads the kept K/V once
// and writes almost nothing, so a copy benchmark (read + write) is not its ceiling; this kernel
// reads a buffer with the same kind of loads the path uses and discards the data.
// Grid-stride 16-byte non-coherent loads (L1 no-allocate, 256-byte L2 prefetch hint), 16 in
// flight per thread, two 1024-thread CTAs per SM. The loaded words are folded into one value that
// is stored only through a pointer the host passes as null, so no load can be elided.
#include "lsa_device.cuh"

namespace lsa {

constexpr int kReadThreads = 1024;
constexpr int kReadU = 16;

// One 16-byte load, folded into `acc`.
template <bool HINT>
__device__ __forceinline__ void touch16(const uint4* p, uint32_t& acc) {
    uint32_t a, b, c, d;
    if (HINT)
        asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(a), "=r"(b), "=r"(c), "=r"(d) : "l"(p));
    else
        asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(a), "=r"(b), "=r"(c), "=r"(d) : "l"(p));
    acc ^= a ^ b ^ c ^ d;
}

__global__ void __launch_bounds__(kReadThreads) k_read_stream(const uint4* __restrict__ buf, size_t n16,
                                                               uint32_t* sink) {
    uint32_t acc = 0;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (; i + (kReadU - 1) * stride < n16; i += kReadU * stride) {
#pragma unroll
        for (int u = 0; u < kReadU; ++u) touch16<true>(buf + i + u * stride, acc);
    }
    for (; i < n16; i += stride) touch16<false>(buf + i, acc);
    if (sink != nullptr) *sink = acc;  // never taken: the host passes null
}

}  // namespace lsa

using namespace lsa;

extern "C" LSA_API lsa_status lsa_read_stream(const void* buf, size_t bytes, void* stream) {
    if (buf == nullptr || bytes == 0 || (reinterpret_cast<uintptr_t>(buf) & 15u) != 0 || (bytes & 15u) != 0)
        return LSA_ERR_INVALID_ARG;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return LSA_ERR_CUDA;
    k_read_stream<<<2 * sms, kReadThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(buf), bytes / 16, nullptr);
    return cudaGetLastError() == cudaSuccess ? LSA_OK : LSA_ERR_CUDA;
}
