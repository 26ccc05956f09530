// shard.cu - the chunk-sharded decode step for sequences split across GPUs.
//
// When one sequence's chunks are spread over G ranks (rank g owns a contiguous run of
// chunks), the LSA step of the review (section 3-2 (3), steps 4-7: score all chunks,
// keep the top-k, attend over the kept chunks) splits into local work and two small
// exchanges:
//   1. each rank scores its chunks and keeps its local top-min(k, n_g) as candidates;
//   2. candidates (score, global chunk id) are all-gathered; since every member of the
//      global top-k is in its own rank's top-k, the top-k of the gathered candidates (same
//      tie rule: lower global id first) is the global keep set;
//   3. each rank attends over the kept chunks it owns and produces (out_g, lse_g);
//   4. the (out, lse) pairs are all-gathered and merged with the log-sum-exp rule:
//      out = sum_g e^(lse_g - M) out_g / sum_g e^(lse_g - M), lse = M + log(sum ...).
// This file holds the kernels of steps 1, 2 and 4 around the existing score, top-k and
// attention kernels; the exchanges are collectives issued by the caller.
#include <cfloat>

#include "lsa_device.cuh"

namespace lsa {

struct ShardOffsets {
    int32_t global0[kMaxB];  // global id of this rank's first chunk, per sequence
};

// grid (B), 256 threads: candidates of one sequence, padded to k_pad with (-FLT_MAX, -1).
__global__ void __launch_bounds__(256)
k_shard_candidates(const float* __restrict__ scores, const int32_t* __restrict__ ids, const SeqTable tab,
                   const ShardOffsets offs, int k_pad, float* __restrict__ cand_scores,
                   int32_t* __restrict__ cand_ids) {
    const int b = blockIdx.x;
    const int kg = tab.kept_off[b + 1] - tab.kept_off[b];
    const int n = tab.chunk_off[b + 1] - tab.chunk_off[b];
    pdl_wait();
    pdl_trigger();
    for (int j = threadIdx.x; j < k_pad; j += blockDim.x) {
        float s = -FLT_MAX;
        int32_t gid = -1;
        if (j < kg) {
            const int32_t id = ids[tab.kept_off[b] + j];
            if (id >= 0 && id < n) {
                s = scores[tab.chunk_off[b] + id];
                gid = offs.global0[b] + id;
            }
        }
        cand_scores[(size_t)b * k_pad + j] = s;
        cand_ids[(size_t)b * k_pad + j] = gid;
    }
}

// grid (B, G): [G][B][k_pad] (all-gather order) -> [B][G][k_pad] (per-sequence order).
__global__ void __launch_bounds__(256)
k_shard_transpose(const float* __restrict__ in_s, const int32_t* __restrict__ in_i, int B, int k_pad,
                  float* __restrict__ out_s, int32_t* __restrict__ out_i) {
    const int b = blockIdx.x, g = blockIdx.y, G = gridDim.y;
    pdl_wait();
    pdl_trigger();
    const size_t src = ((size_t)g * B + b) * k_pad, dst = ((size_t)b * G + g) * k_pad;
    for (int j = threadIdx.x; j < k_pad; j += blockDim.x) {
        out_s[dst + j] = in_s[src + j];
        out_i[dst + j] = in_i[src + j];
    }
}

// grid (B), 256 threads: the global keep positions of sequence b (ascending positions in
// [0, G*k_pad), i.e. ascending global ids) -> global ids, and this rank's local ids + count.
__global__ void __launch_bounds__(256)
k_shard_select(const int32_t* __restrict__ pos, const int32_t* __restrict__ cand_ids, const SeqTable gtab,
               const ShardOffsets offs, const SeqTable ltab, int G, int k_pad, int32_t* __restrict__ local_ids,
               int32_t* __restrict__ local_count, int32_t* __restrict__ global_ids) {
    __shared__ int32_t s_count;
    const int b = blockIdx.x;
    const int k = gtab.kept_off[b + 1] - gtab.kept_off[b];
    const int lo = offs.global0[b];
    const int hi = lo + (ltab.chunk_off[b + 1] - ltab.chunk_off[b]);
    pdl_wait();
    pdl_trigger();
    if (threadIdx.x == 0) s_count = 0;
    __syncthreads();
    // positions are ascending, so this rank's kept ids form one contiguous run of them
    for (int j = threadIdx.x; j < k; j += blockDim.x) {
        const int p = pos[gtab.kept_off[b] + j];
        const int32_t gid = (p >= 0 && p < G * k_pad) ? cand_ids[(size_t)b * G * k_pad + p] : -1;
        if (global_ids) global_ids[gtab.kept_off[b] + j] = gid;
        if (gid >= lo && gid < hi) atomicAdd(&s_count, 1);
    }
    __syncthreads();
    const int count = s_count;
    // first kept position owned by this rank: the number of kept ids below `lo`
    __shared__ int32_t s_first;
    if (threadIdx.x == 0) s_first = 0;
    __syncthreads();
    for (int j = threadIdx.x; j < k; j += blockDim.x) {
        const int p = pos[gtab.kept_off[b] + j];
        const int32_t gid = (p >= 0 && p < G * k_pad) ? cand_ids[(size_t)b * G * k_pad + p] : -1;
        if (gid >= 0 && gid < lo) atomicAdd(&s_first, 1);
    }
    __syncthreads();
    const int first = s_first;
    const int cap = ltab.kept_off[b + 1] - ltab.kept_off[b];
    for (int j = threadIdx.x; j < cap; j += blockDim.x) {
        int32_t v = -1;
        if (j < count) {
            const int p = pos[gtab.kept_off[b] + first + j];
            v = cand_ids[(size_t)b * G * k_pad + p] - lo;
        }
        local_ids[ltab.kept_off[b] + j] = v;
    }
    if (threadIdx.x == 0) local_count[b] = min(count, cap);
}

// grid (B, H), Dh threads: log-sum-exp merge of G ranks' normalised outputs.
__global__ void __launch_bounds__(kDh)
k_merge_partials(const float* __restrict__ outs, const float* __restrict__ lses, int G, int B, int H,
                 float* __restrict__ out, float* __restrict__ lse) {
    const int b = blockIdx.x, h = blockIdx.y, d = threadIdx.x;
    pdl_wait();
    pdl_trigger();
    float M = -INFINITY;
    for (int g = 0; g < G; ++g) M = fmaxf(M, lses[((size_t)g * B + b) * H + h]);
    float L = 0.f, A = 0.f;
    if (M != -INFINITY) {
        for (int g = 0; g < G; ++g) {
            const float lg = lses[((size_t)g * B + b) * H + h];
            if (lg == -INFINITY) continue;  // a rank that kept nothing
            const float wgt = expf(lg - M);
            L += wgt;
            A = fmaf(wgt, outs[(((size_t)g * B + b) * H + h) * kDh + d], A);
        }
    }
    out[((size_t)b * H + h) * kDh + d] = L > 0.f ? A / L : 0.f;
    if (lse != nullptr && d == 0) lse[(size_t)b * H + h] = L > 0.f ? M + logf(L) : -INFINITY;
}

cudaError_t launch_shard_candidates(const SeqTable& tab, int B, const ShardOffsets& offs, int k_pad,
                                    const float* scores, const int32_t* ids, float* cs, int32_t* ci,
                                    cudaStream_t st) {
    k_shard_candidates<<<B, 256, 0, st>>>(scores, ids, tab, offs, k_pad, cs, ci);
    return cudaGetLastError();
}

cudaError_t launch_shard_transpose(int G, int B, int k_pad, const float* in_s, const int32_t* in_i, float* out_s,
                                   int32_t* out_i, cudaStream_t st) {
    k_shard_transpose<<<dim3(B, G), 256, 0, st>>>(in_s, in_i, B, k_pad, out_s, out_i);
    return cudaGetLastError();
}

cudaError_t launch_shard_select(const int32_t* pos, const int32_t* cand_ids, const SeqTable& gtab,
                                const ShardOffsets& offs, const SeqTable& ltab, int B, int G, int k_pad,
                                int32_t* local_ids, int32_t* local_count, int32_t* global_ids, cudaStream_t st) {
    k_shard_select<<<B, 256, 0, st>>>(pos, cand_ids, gtab, offs, ltab, G, k_pad, local_ids, local_count, global_ids);
    return cudaGetLastError();
}

cudaError_t launch_merge_partials(const float* outs, const float* lses, int G, int B, int H, float* out, float* lse,
                                  cudaStream_t st) {
    k_merge_partials<<<dim3(B, H), kDh, 0, st>>>(outs, lses, G, B, H, out, lse);
    return cudaGetLastError();
}

}  // namespace lsa
