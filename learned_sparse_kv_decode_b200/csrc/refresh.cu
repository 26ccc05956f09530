// refresh.cu - incremental refresh of the resident KV set at a retrieval cycle.
//
// FlashMemory-DeepSeek-V4 (review on dimensionstp.github.io, section 3-1 table
// "Retrieval interval: re-score about every 64 decode steps", and section 3-2 (3),
// steps 4-7): at each retrieval cycle the indexer re-scores every chunk and a new
// keep set is chosen; until the next cycle, attention runs over the resident
// chunks. Only the query-critical chunks stay resident (arXiv abstract).
//
// Resident buffer: k_b slots per sequence; slot j of sequence b holds the C token
// rows of chunk slot_ids[kept_off[b] + j] (or is empty, id -1). A refresh makes the
// resident set equal to the new top-k set while moving as little as possible:
//   * a slot whose chunk stays in the set keeps it (no copy);
//   * the other slots are freed; the entering chunks, in ascending chunk order, fill the
//     freed slots in ascending slot order, and only they are copied.
// k_refresh_plan computes that assignment (one CTA per sequence, bitmaps in shared
// memory, block scans for the two ascending orders); k_refresh_copy copies the
// entering chunks' K and V rows.
#include "lsa_device.cuh"

namespace lsa {

constexpr int kPlanThreads = 1024;
constexpr int kPlanWarps = kPlanThreads / 32;
constexpr int kRefreshMaxChunks = 1 << 19;  // two bitmaps of 64 KiB per CTA

// Block-wide exclusive scan of one 0/1 flag per thread; returns the prefix and the tile total.
__device__ __forceinline__ uint32_t block_excl_scan_flag(bool f, uint32_t* warp_tot, uint32_t& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t ball = __ballot_sync(0xffffffffu, f);
    if (lane == 0) warp_tot[warp] = __popc(ball);
    __syncthreads();
    uint32_t before = __popc(ball & ((1u << lane) - 1u)), tot = 0;
    for (int w = 0; w < kPlanWarps; ++w) {
        const uint32_t t = warp_tot[w];
        if (w < warp) before += t;
        tot += t;
    }
    __syncthreads();  // warp_tot is reused by the next tile
    total = tot;
    return before;
}

// grid (B), 1024 threads; dynamic smem: two bitmaps of ceil(max_n / 32) words.
// new_ids: this cycle's top-k ids (ascending); slot_ids: in/out slot table.
// copy_src / copy_dst: per sequence, the entering chunk ids and their slots (capacity k_b);
// copy_count[b]: how many entries are valid; moved (nullable): same count, for the caller.
__global__ void __launch_bounds__(kPlanThreads)
k_refresh_plan(const int32_t* __restrict__ new_ids, int32_t* __restrict__ slot_ids,
               int32_t* __restrict__ copy_src, int32_t* __restrict__ copy_dst,
               int32_t* __restrict__ copy_count, int32_t* __restrict__ moved, const SeqTable tab,
               int words) {
    extern __shared__ uint32_t bits[];  // [0, words): in the new set; [words, 2 words): stays resident
    __shared__ uint32_t warp_tot[kPlanWarps];
    uint32_t* in_new = bits;
    uint32_t* stays = bits + words;
    const int b = blockIdx.x, tid = threadIdx.x;
    const int n = tab.chunk_off[b + 1] - tab.chunk_off[b];
    const int k = tab.kept_off[b + 1] - tab.kept_off[b];
    const int32_t* nid = new_ids + tab.kept_off[b];
    int32_t* slots = slot_ids + tab.kept_off[b];
    pdl_wait();
    pdl_trigger();

    const int wn = (n + 31) / 32;
    for (int i = tid; i < 2 * words; i += kPlanThreads) bits[i] = 0;
    __syncthreads();
    for (int j = tid; j < k; j += kPlanThreads) {
        const int c = nid[j];
        if (c >= 0 && c < n) atomicOr(&in_new[c >> 5], 1u << (c & 31));
    }
    __syncthreads();
    // slots whose chunk stays keep it; mark those chunks as already resident. A chunk listed
    // in two slots (a corrupt table) stays in one of them (whichever claims it first); the
    // others are emptied, so the set never holds a chunk twice.
    for (int j = tid; j < k; j += kPlanThreads) {
        const int c = slots[j];
        if (c >= 0 && c < n && (in_new[c >> 5] >> (c & 31) & 1u)) {
            const uint32_t bit = 1u << (c & 31);
            if (atomicOr(&stays[c >> 5], bit) & bit) slots[j] = -1;
        }
    }
    __syncthreads();
    (void)wn;

    // entering chunks (in the new set, not resident) in ascending order -> rank
    // freed slots (empty, or holding a chunk that left) in ascending slot order -> rank
    uint32_t enter_base = 0, free_base = 0;
    int32_t* src = copy_src + tab.kept_off[b];
    int32_t* dst = copy_dst + tab.kept_off[b];
    for (int j0 = 0; j0 < k; j0 += kPlanThreads) {
        const int j = j0 + tid;
        bool entering = false;
        int c = -1;
        if (j < k) {
            c = nid[j];
            entering = c >= 0 && c < n && !(stays[c >> 5] >> (c & 31) & 1u);
        }
        uint32_t tot;
        const uint32_t r = enter_base + block_excl_scan_flag(entering, warp_tot, tot);
        if (entering) src[r] = c;
        enter_base += tot;
    }
    for (int j0 = 0; j0 < k; j0 += kPlanThreads) {
        const int j = j0 + tid;
        bool freed = false;
        if (j < k) {
            const int c = slots[j];
            freed = !(c >= 0 && c < n && (stays[c >> 5] >> (c & 31) & 1u));
        }
        uint32_t tot;
        const uint32_t r = free_base + block_excl_scan_flag(freed, warp_tot, tot);
        if (freed) dst[r] = j;
        free_base += tot;
    }
    __syncthreads();  // src[] and dst[] complete before the slot table is rewritten
    // both counts equal k minus the chunks that stay (min() only guards the buffers)
    const uint32_t moves = min(enter_base, free_base);
    for (uint32_t r = tid; r < moves; r += kPlanThreads) slots[dst[r]] = src[r];
    if (tid == 0) {
        copy_count[b] = (int32_t)moves;
        if (moved) moved[b] = (int32_t)moves;
    }
}

// grid (sum k_b, 2): entry j of the copy list, K (y = 0) or V (y = 1).
__global__ void __launch_bounds__(512)
k_refresh_copy(const uint8_t* __restrict__ K, const uint8_t* __restrict__ V,
               uint8_t* __restrict__ K_res, uint8_t* __restrict__ V_res,
               const int32_t* __restrict__ copy_src, const int32_t* __restrict__ copy_dst,
               const int32_t* __restrict__ copy_count, const SeqTable tab, uint64_t chunk_bytes) {
    const int j = blockIdx.x;
    const int b = seq_of(tab.kept_off, tab.B, j);
    pdl_wait();
    pdl_trigger();
    const int r = j - tab.kept_off[b];
    if (r >= copy_count[b]) return;
    const int c = copy_src[j], slot = copy_dst[j];
    const uint8_t* s = (blockIdx.y ? V : K) + ((uint64_t)tab.chunk_off[b] + (uint64_t)c) * chunk_bytes;
    uint8_t* d = (blockIdx.y ? V_res : K_res) + ((uint64_t)tab.kept_off[b] + (uint64_t)slot) * chunk_bytes;
    const uint64_t nvec = chunk_bytes / 16;
    for (uint64_t v0 = threadIdx.x; v0 < nvec; v0 += 512 * 8) {
        uint4 x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const uint64_t v = v0 + (uint64_t)u * 512;
            if (v < nvec) x[u] = ld_stream16(s + v * 16);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const uint64_t v = v0 + (uint64_t)u * 512;
            if (v < nvec) st_stream16(d + v * 16, x[u]);
        }
    }
}

cudaError_t refresh_init_attrs() {
    cudaError_t e = set_smem_attrs(k_refresh_plan, 2 * (kRefreshMaxChunks / 32) * 4);
    if (e == cudaSuccess) e = set_smem_attrs(k_refresh_copy, 0);
    return e;
}

size_t refresh_smem(int max_n) { return (size_t)2 * ((max_n + 31) / 32) * 4; }

int refresh_max_chunks() { return kRefreshMaxChunks; }

cudaError_t launch_refresh(const lsa_dims& d, const SeqTable& tab, int max_n, const int32_t* new_ids,
                           int32_t* slot_ids, const void* K, const void* V, void* K_res, void* V_res,
                           int32_t* copy_src, int32_t* copy_dst, int32_t* copy_count, int32_t* moved,
                           cudaStream_t stream) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(d.B, 1, 1);
    cfg.blockDim = dim3(kPlanThreads, 1, 1);
    const int words = (max_n + 31) / 32;
    cfg.dynamicSmemBytes = refresh_smem(max_n);
    cudaError_t e = cudaLaunchKernelEx(&cfg, k_refresh_plan, new_ids, slot_ids, copy_src, copy_dst,
                                       copy_count, moved, tab, words);
    if (e != cudaSuccess) return e;
    const int es = d.kv_dtype == LSA_BF16 ? 2 : 4;
    const uint64_t chunk_bytes = (uint64_t)d.chunk_len * d.H * d.Dh * es;
    cudaLaunchConfig_t ccfg = {};
    ccfg.stream = stream;
    ccfg.attrs = attr;
    ccfg.numAttrs = 1;
    ccfg.gridDim = dim3(tab.kept_off[d.B], 2, 1);
    ccfg.blockDim = dim3(512, 1, 1);
    return cudaLaunchKernelEx(&ccfg, k_refresh_copy, (const uint8_t*)K, (const uint8_t*)V, (uint8_t*)K_res,
                              (uint8_t*)V_res, (const int32_t*)copy_src, (const int32_t*)copy_dst,
                              (const int32_t*)copy_count, tab, chunk_bytes);
}

}  // namespace lsa
