// lsa_device.cuh - device-side helpers shared by the LSA kernels (sm_100a):
// launch plans passed by value, bf16 unpacking, mbarriers, 1-D bulk copies,
// programmatic dependent launch, bounded waits and the sticky error word.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/lsa.h"

namespace lsa {

// Sticky device error bits (first word of the workspace).
enum : uint32_t {
    kErrNonFinite = 1u << 0,
    kErrBadId = 1u << 1,
    kErrTimeout = 1u << 2,
};

constexpr int kDh = LSA_HEAD_DIM;
constexpr int kMaxB = LSA_MAX_BATCH;
constexpr size_t kWsHeader = 256;  // bytes reserved at the start of the workspace

// Per-call sequence table, passed by value as a kernel parameter (about 3 KB).
struct SeqTable {
    int32_t B;
    int32_t C;                   // tokens per chunk
    int32_t chunk_off[kMaxB + 1];  // prefix of N_b over the flattened chunk axis
    int32_t kept_off[kMaxB + 1];   // prefix of k_b over the flattened id axis
};

// ---------------------------------------------------------------- small helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void set_error(uint32_t* err, uint32_t bits) {
    if (err) atomicOr(err, bits);
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Two bf16 packed in a 32-bit word -> two floats (exact widening).
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// 16-byte streaming load that does not allocate in L1.
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void st_stream16(void* p, uint4 v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

// ---------------------------------------------------------------- PDL
// Wait until the preceding kernel in the stream (launched with programmatic
// stream serialisation) has completed and its writes are visible.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Allow the next kernel in the stream to start launching.
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- mbarriers
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase of `parity` to complete: gives up after
// kWaitLimitNs of wall time (or 2^26 polls), records kErrTimeout, returns false.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint32_t* err) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t i = 0; i < (1u << 26); ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 255u && global_timer_ns() - t0 > kWaitLimitNs) break;
    }
    set_error(err, kErrTimeout);
    return false;
}

// ---------------------------------------------------------------- 1-D bulk copy (TMA engine)
// Global -> this CTA's shared memory; completion is signalled on `bar` as tx bytes.
// Both addresses 16-byte aligned, bytes a multiple of 16. No cluster multicast.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// Dynamic shared-memory limit plus the maximum shared-memory carveout, so consecutive
// kernels of a step do not make the SM switch its L1 / shared-memory split.
template <typename Kernel>
inline cudaError_t set_smem_attrs(Kernel* kernel, int max_dynamic_smem) {
    cudaError_t e = cudaSuccess;
    if (max_dynamic_smem > 0)
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, max_dynamic_smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
    return e;
}

// Sequence of a flattened position `i` given a prefix table (binary search).
__device__ __forceinline__ int seq_of(const int32_t* off, int B, int64_t i) {
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (off[mid] <= i) lo = mid; else hi = mid - 1;
    }
    return lo;
}

}  // namespace lsa
