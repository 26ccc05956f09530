// Test-only kernel: the library's bounded mbarrier wait, run on a barrier that nothing ever
// arrives on. The wait must give up after its time limit, record the timeout bit in the sticky
// error word and return, leaving the CUDA context usable. No fault, trap or endless loop.
#include <cuda_runtime.h>

#include "../../learned_sparse_kv_decode_b200/csrc/lsa_device.cuh"

__global__ void k_wait_forever_bounded(uint32_t* err, unsigned long long* elapsed_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        lsa::mbar_init(lsa::smem_u32(&bar), 1);  // expects one arrival that never comes
        lsa::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint64_t t0 = lsa::global_timer_ns();
        const bool ok = lsa::mbar_wait(lsa::smem_u32(&bar), 0, err);
        elapsed_ns[0] = lsa::global_timer_ns() - t0;
        elapsed_ns[1] = ok ? 1ull : 0ull;
    }
}

extern "C" __attribute__((visibility("default"))) int wt_run(void* err_word, void* elapsed_ns) {
    k_wait_forever_bounded<<<1, 32>>>(static_cast<uint32_t*>(err_word), static_cast<unsigned long long*>(elapsed_ns));
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    return (int)e;
}
