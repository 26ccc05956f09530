// gather.cu - compaction of the kept chunks' K/V into a resident buffer.
//
// FlashMemory-DeepSeek-V4 (arXiv abstract; review on dimensionstp.github.io,
// section 3-2 (3), step 6): only the query-critical KV chunks stay resident in
// GPU memory. This kernel copies, for every kept chunk j of sequence b, the C
// token rows [ids[j]*C, ids[j]*C + C) of its K and V caches to rows
// [j*C, j*C + C) of the sequence's block of K_res / V_res. A chunk of C tokens
// x H heads x Dh is one contiguous run in both buffers, so this is a pure
// streaming copy with 128-bit loads and stores.
#include "lsa_device.cuh"

namespace lsa {

constexpr int kGatherThreads = 512;
constexpr int kGatherUnroll = 8;

// grid (sum k_b, 2): blockIdx.y selects K (0) or V (1).
__global__ void __launch_bounds__(kGatherThreads)
k_gather(const uint8_t* __restrict__ K, const uint8_t* __restrict__ V,
         const int32_t* __restrict__ ids, uint8_t* __restrict__ K_res, uint8_t* __restrict__ V_res,
         const SeqTable tab, uint64_t chunk_bytes, uint32_t* err) {
    const int j = blockIdx.x;
    const int b = seq_of(tab.kept_off, tab.B, j);
    const int n_b = tab.chunk_off[b + 1] - tab.chunk_off[b];
    pdl_wait();
    pdl_trigger();
    const int32_t id = ids[j];
    if (id < 0 || id >= n_b) {
        if (threadIdx.x == 0) set_error(err, kErrBadId);
        return;
    }
    const uint8_t* src = (blockIdx.y ? V : K) + ((uint64_t)tab.chunk_off[b] + (uint64_t)id) * chunk_bytes;
    uint8_t* dst = (blockIdx.y ? V_res : K_res) + (uint64_t)j * chunk_bytes;
    const uint64_t nvec = chunk_bytes / 16;
    const uint64_t step = (uint64_t)kGatherThreads * kGatherUnroll;
    for (uint64_t v0 = threadIdx.x; v0 < nvec; v0 += step) {
        uint4 x[kGatherUnroll];
#pragma unroll
        for (int u = 0; u < kGatherUnroll; ++u) {
            const uint64_t v = v0 + (uint64_t)u * kGatherThreads;
            if (v < nvec) x[u] = ld_stream16(src + v * 16);
        }
#pragma unroll
        for (int u = 0; u < kGatherUnroll; ++u) {
            const uint64_t v = v0 + (uint64_t)u * kGatherThreads;
            if (v < nvec) st_stream16(dst + v * 16, x[u]);
        }
    }
}

cudaError_t launch_gather(const lsa_dims& d, const SeqTable& tab, const void* K, const void* V,
                          const int32_t* ids, void* K_res, void* V_res, uint32_t* err,
                          cudaStream_t stream) {
    const int es = d.kv_dtype == LSA_BF16 ? 2 : 4;
    const uint64_t chunk_bytes = (uint64_t)d.chunk_len * d.H * d.Dh * es;
    cudaLaunchConfig_t cfg = {};
    cfg.stream = stream;
    cfg.gridDim = dim3(tab.kept_off[d.B], 2, 1);
    cfg.blockDim = dim3(kGatherThreads, 1, 1);
    return cudaLaunchKernelEx(&cfg, k_gather, (const uint8_t*)K, (const uint8_t*)V, ids,
                              (uint8_t*)K_res, (uint8_t*)V_res, tab, chunk_bytes, err);
}

}  // namespace lsa
