// small.cu - the whole decode step in one launch, for a few short sequences.
//
// FlashMemory-DeepSeek-V4 (review on dimensionstp.github.io, section 3-2 (3), steps 4-7): score
// every chunk, keep the top-k, attend over the kept chunks only. For a few short sequences the
// four kernels of the general path (score, top-k, split attention, merge) are bound by their
// launches, not by the bytes they move. k_decode_small does the four steps in one grid:
//  * CTA (j, h, b) recomputes the scores of sequence b (at most kSmallMaxN chunks; after the
//    first CTA they come from L2) and ranks them: a chunk is kept when fewer than k_b chunks come
//    before it in the order (score desc, index asc), so the kept set is the top-k with ties to the
//    lower index. A block scan lists the kept ids in ascending order; CTA (0, 0, b) writes them.
//  * It then attends head h over the j-th kept chunk (fp32 online softmax in the log2 domain,
//    one warp per token group, warps combined in shared memory) and writes an unnormalised
//    partial (acc, m, l) to the workspace.
//  * When k_b <= 8 for every sequence, the k_b CTAs of (b, h) form one thread-block cluster:
//    each keeps its partial in shared memory, and after a cluster barrier CTA 0 of the cluster
//    reads them through distributed shared memory and merges them in kept order. Otherwise the
//    partials go to the workspace and the last of the k_b CTAs to finish (an arrival counter in
//    the workspace header, reset by that CTA) merges them. Either way the merge order is the
//    kept order, so the result is deterministic.
#include <algorithm>
#include <cmath>

#include "lsa_device.cuh"

namespace lsa {

constexpr int kSmallThreads = 256;
constexpr int kSmallWarps = kSmallThreads / 32;
constexpr int kSmallMaxN = 256;      // chunks per sequence
constexpr int kSmallCounters = 48;   // (sequence, head) pairs: header words 16..63
constexpr size_t kSmallCounterOff = 64;  // byte offset of the counters in the workspace header
constexpr int kSmallUnroll = 8;      // rows (scores) or tokens (attention) in flight per warp
constexpr int kSmallMaxCluster = 8;  // k_b up to this: the CTAs of (b, h) merge inside a cluster

__device__ __forceinline__ void small_cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// A float of the shared memory of CTA `rank` of this cluster, at the offset of `p`.
__device__ __forceinline__ float small_dsmem_ld(const float* p, uint32_t rank) {
    uint32_t remote;
    float v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(p)), "r"(rank));
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}

// Order-preserving map float -> uint32 (larger float -> larger key); -0 maps like +0; NaN maps
// to 0 (never preferred). Non-finite scores set `bad`.
__device__ __forceinline__ uint32_t small_key(float f, bool& bad) {
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7F800000u) == 0x7F800000u) {
        bad = true;
        if (u & 0x007FFFFFu) return 0u;
    }
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <bool BF16>
__device__ __forceinline__ void small_unpack(const uint4& v, float (&x)[8]) {
    if constexpr (BF16) {
        x[0] = bf16lo(v.x); x[1] = bf16hi(v.x); x[2] = bf16lo(v.y); x[3] = bf16hi(v.y);
        x[4] = bf16lo(v.z); x[5] = bf16hi(v.z); x[6] = bf16lo(v.w); x[7] = bf16hi(v.w);
    } else {
        x[0] = __uint_as_float(v.x); x[1] = __uint_as_float(v.y);
        x[2] = __uint_as_float(v.z); x[3] = __uint_as_float(v.w);
        x[4] = x[5] = x[6] = x[7] = 0.f;
    }
}

__device__ __forceinline__ float small_ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// grid (max k_b, H, B), kSmallThreads threads; with CL, clusters of (max k_b, 1, 1).
// EBF16: embeddings are bf16 (else fp32); KBF16: q, K, V are bf16 (else fp32).
template <bool EBF16, bool KBF16, bool CL>
__global__ void __launch_bounds__(kSmallThreads)
k_decode_small(const uint8_t* __restrict__ q_emb, const uint8_t* __restrict__ emb,
               const uint8_t* __restrict__ q, const uint8_t* __restrict__ K, const uint8_t* __restrict__ V,
               int32_t* __restrict__ ids_out, float* __restrict__ out, float* __restrict__ lse,
               float* __restrict__ part, const SeqTable tab, int E, int H, float qscale, uint32_t* ws) {
    constexpr int EES = EBF16 ? 2 : 4;
    constexpr int EVEC = 16 / EES;  // embedding elements per 16-byte piece
    constexpr int KES = KBF16 ? 2 : 4;
    constexpr int KVEC = 16 / KES;  // head-dim elements per lane
    constexpr int LPH = kDh / KVEC; // lanes per token row (32 fp32, 16 bf16)
    constexpr int TPW = 32 / LPH;   // tokens per warp step
    __shared__ uint32_t s_key[kSmallMaxN];
    __shared__ int32_t s_kept[kSmallMaxN];
    __shared__ uint32_t s_wcount[kSmallWarps];
    __shared__ float s_part[kSmallWarps * TPW][kDh + 2];
    __shared__ float s_fin[kDh + 2];  // this CTA's partial (acc, m, l), read by the cluster
    __shared__ int s_last;

    const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n = tab.chunk_off[b + 1] - tab.chunk_off[b];
    const int kb = tab.kept_off[b + 1] - tab.kept_off[b];
    if (!CL && j >= kb) return;  // the whole CTA: grid x covers the largest k_b
    if (j < kb) {  // (in a cluster every CTA reaches the cluster barriers below)

        // ---- 1. scores of sequence b: one row per warp step, lane l holds the 16-byte piece l
        const int P = E / EVEC;  // pieces per row, <= 32
        const uint32_t row_bytes = (uint32_t)E * EES;
        float qe[8];
        {
            uint4 t = make_uint4(0u, 0u, 0u, 0u);
            if (lane < P) t = *reinterpret_cast<const uint4*>(q_emb + (size_t)b * row_bytes + (size_t)lane * 16);
            small_unpack<EBF16>(t, qe);
        }
        const uint8_t* rows = emb + (size_t)tab.chunk_off[b] * row_bytes;
        bool bad = false;
        for (int r0 = warp; r0 < n; r0 += kSmallWarps * kSmallUnroll) {
            float acc[kSmallUnroll];
#pragma unroll
            for (int u = 0; u < kSmallUnroll; ++u) {
                const int r = r0 + u * kSmallWarps;
                uint4 t = make_uint4(0u, 0u, 0u, 0u);
                if (r < n && lane < P) t = ld_stream16(rows + (size_t)r * row_bytes + (size_t)lane * 16);
                float x[8];
                small_unpack<EBF16>(t, x);
                float a = 0.f;
#pragma unroll
                for (int e = 0; e < EVEC; ++e) a = fmaf(qe[e], x[e], a);
                acc[u] = a;
            }
#pragma unroll
            for (int u = 0; u < kSmallUnroll; ++u)
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], off);
            if (lane == 0) {
#pragma unroll
                for (int u = 0; u < kSmallUnroll; ++u) {
                    const int r = r0 + u * kSmallWarps;
                    if (r < n) s_key[r] = small_key(acc[u], bad);
                }
            }
        }
        if (bad && j == 0 && h == 0) set_error(ws, kErrNonFinite);
        __syncthreads();

        // ---- 2. the kept set: chunk i is kept when fewer than k_b chunks come before it
        bool kept = false;
        if (tid < n) {
            const uint32_t ki = s_key[tid];
            int before = 0;
            for (int c = 0; c < n; ++c) {
                const uint32_t kc = s_key[c];
                before += (kc > ki || (kc == ki && c < tid)) ? 1 : 0;
            }
            kept = before < kb;
        }
        const uint32_t ball = __ballot_sync(0xffffffffu, kept);
        if (lane == 0) s_wcount[warp] = __popc(ball);
        __syncthreads();
        if (kept) {
            int pos = __popc(ball & ((1u << lane) - 1u));
            for (int w = 0; w < warp; ++w) pos += s_wcount[w];
            s_kept[pos] = tid;
        }
        __syncthreads();
        if (j == 0 && h == 0)
            for (int p = tid; p < kb; p += kSmallThreads) ids_out[tab.kept_off[b] + p] = s_kept[p];

        // ---- 3. attention of head h over kept chunk j: TPW token groups per warp, LPH lanes each
        const int C = tab.C;
        const int sub = lane / LPH, li = lane % LPH;
        const uint64_t tok_stride = (uint64_t)H * kDh * KES;
        const uint8_t* kbase = K + ((uint64_t)(tab.chunk_off[b] + s_kept[j]) * C) * tok_stride + (uint64_t)h * kDh * KES;
        const uint8_t* vbase = V + ((uint64_t)(tab.chunk_off[b] + s_kept[j]) * C) * tok_stride + (uint64_t)h * kDh * KES;
        float qf[8];
        {
            const uint4 t = *reinterpret_cast<const uint4*>(q + ((uint64_t)b * H + h) * kDh * KES + (uint64_t)li * 16);
            small_unpack<KBF16>(t, qf);
#pragma unroll
            for (int e = 0; e < 8; ++e) qf[e] *= qscale;
        }
        float m = -INFINITY, l = 0.f, o[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = 0.f;
        const int tstep = kSmallWarps * TPW;
        for (int t0 = warp * TPW + sub; t0 < C; t0 += tstep * kSmallUnroll) {
            uint4 kv[kSmallUnroll], vv[kSmallUnroll];
#pragma unroll
            for (int u = 0; u < kSmallUnroll; ++u) {
                const int t = t0 + u * tstep;
                kv[u] = vv[u] = make_uint4(0u, 0u, 0u, 0u);
                if (t < C) {
                    kv[u] = ld_stream16(kbase + (uint64_t)t * tok_stride + (uint64_t)li * 16);
                    vv[u] = ld_stream16(vbase + (uint64_t)t * tok_stride + (uint64_t)li * 16);
                }
            }
            float s[kSmallUnroll];
#pragma unroll
            for (int u = 0; u < kSmallUnroll; ++u) {
                float x[8];
                small_unpack<KBF16>(kv[u], x);
                float a = 0.f;
#pragma unroll
                for (int e = 0; e < KVEC; ++e) a = fmaf(qf[e], x[e], a);
#pragma unroll
                for (int off = LPH >> 1; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
                s[u] = t0 + u * tstep < C ? a : -INFINITY;
            }
            float mx = m;
#pragma unroll
            for (int u = 0; u < kSmallUnroll; ++u) mx = fmaxf(mx, s[u]);
            if (mx == -INFINITY) continue;  // every token of this step is past the chunk (uniform per group)
            const float corr = m == -INFINITY ? 0.f : small_ex2(m - mx);
            l *= corr;
#pragma unroll
            for (int e = 0; e < 8; ++e) o[e] *= corr;
#pragma unroll
            for (int u = 0; u < kSmallUnroll; ++u) {
                const float p = s[u] == -INFINITY ? 0.f : small_ex2(s[u] - mx);
                l += p;
                float x[8];
                small_unpack<KBF16>(vv[u], x);
#pragma unroll
                for (int e = 0; e < KVEC; ++e) o[e] = fmaf(p, x[e], o[e]);
            }
            m = mx;
        }
        // combine the token groups of the CTA, then write this chunk's partial (acc[Dh], m, l)
        {
            float* mine = s_part[warp * TPW + sub];
#pragma unroll
            for (int e = 0; e < KVEC; ++e) mine[li * KVEC + e] = o[e];
            if (li == 0) {
                mine[kDh] = m;
                mine[kDh + 1] = l;
            }
        }
        __syncthreads();
        if (tid < kDh) {
            float M = -INFINITY;
            for (int g = 0; g < tstep; ++g) M = fmaxf(M, s_part[g][kDh]);
            float A = 0.f, L = 0.f;
            for (int g = 0; g < tstep; ++g) {
                const float w = s_part[g][kDh] == -INFINITY ? 0.f : small_ex2(s_part[g][kDh] - M);
                A = fmaf(w, s_part[g][tid], A);
                L = fmaf(w, s_part[g][kDh + 1], L);
            }
            if constexpr (CL) {
                s_fin[tid] = A;
                if (tid == 0) {
                    s_fin[kDh] = M;
                    s_fin[kDh + 1] = L;
                }
            } else {
                float* my_part = part + (((int64_t)tab.kept_off[b] + j) * H + h) * (kDh + 2);
                my_part[tid] = A;
                if (tid == 0) {
                    my_part[kDh] = M;
                    my_part[kDh + 1] = L;
                }
            }
        }
    }  // j < kb

    // ---- 4. merge of the k_b partials of (b, h) in kept order
    if constexpr (CL) {
        small_cluster_sync();  // every partial of the cluster is in its CTA's shared memory
        if (j == 0 && tid < kDh) {
            float M = -INFINITY;
            for (int c = 0; c < kb; ++c) M = fmaxf(M, small_dsmem_ld(&s_fin[kDh], (uint32_t)c));
            float A = 0.f, L = 0.f;
            for (int c = 0; c < kb; ++c) {
                const float mc = small_dsmem_ld(&s_fin[kDh], (uint32_t)c);
                const float w = mc == -INFINITY ? 0.f : small_ex2(mc - M);
                A = fmaf(w, small_dsmem_ld(&s_fin[tid], (uint32_t)c), A);
                L = fmaf(w, small_dsmem_ld(&s_fin[kDh + 1], (uint32_t)c), L);
            }
            out[((int64_t)b * H + h) * kDh + tid] = L > 0.f ? A / L : 0.f;
            if (lse != nullptr && tid == 0) lse[(int64_t)b * H + h] = (M + log2f(L)) * 0.69314718055994531f;
        }
        small_cluster_sync();  // every CTA's shared memory stays alive until CTA 0 has read it
        return;
    }
    __syncthreads();
    uint32_t* counter = ws + kSmallCounterOff / 4 + (b * H + h);
    if (tid == 0) {
        __threadfence();  // this CTA's partial is visible before it is counted
        const uint32_t before = atomicAdd(counter, 1u);
        s_last = before == (uint32_t)(kb - 1) ? 1 : 0;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const float* p0 = part + ((int64_t)tab.kept_off[b] * H + h) * (kDh + 2);
    const int64_t pstride = (int64_t)H * (kDh + 2);
    if (tid < kDh) {
        float M = -INFINITY;
        for (int c = 0; c < kb; ++c) M = fmaxf(M, __ldcg(p0 + c * pstride + kDh));
        float A = 0.f, L = 0.f;
        for (int c = 0; c < kb; ++c) {
            const float* pc = p0 + c * pstride;
            const float mc = __ldcg(pc + kDh);
            const float w = mc == -INFINITY ? 0.f : small_ex2(mc - M);
            A = fmaf(w, __ldcg(pc + tid), A);
            L = fmaf(w, __ldcg(pc + kDh + 1), L);
        }
        out[((int64_t)b * H + h) * kDh + tid] = L > 0.f ? A / L : 0.f;
        if (lse != nullptr && tid == 0) lse[(int64_t)b * H + h] = (M + log2f(L)) * 0.69314718055994531f;
        if (tid == 0) *counter = 0u;  // every CTA of (b, h) has arrived: ready for the next call
    }
}

// ------------------------------------------------------------------ host side
// The one-launch step serves: one query per sequence, at most kSmallCounters (sequence, head)
// pairs, at most kSmallMaxN chunks per sequence, embedding rows of at most 512 bytes, and at
// most `max_kv_bytes` of kept K/V (beyond that the split attention streams them better). Its
// partials (total_kept * H rows of Dh + 2 floats) have a workspace region of their own.
bool small_step_eligible(const lsa_dims& d, int max_n, int64_t total_kept) {
    const int es = d.emb_dtype == LSA_BF16 ? 2 : 4;
    const int kvs = d.kv_dtype == LSA_BF16 ? 2 : 4;
    if (d.Q != 1 || d.B * d.H > kSmallCounters || max_n > kSmallMaxN) return false;
    if (d.E * es > 512 || (d.E * es) % 16 != 0) return false;
    const int64_t kv_bytes = total_kept * (int64_t)d.chunk_len * d.H * kDh * kvs * 2;
    constexpr int64_t max_kv_bytes = (int64_t)16 << 20;
    return kv_bytes <= max_kv_bytes;
}

size_t small_step_part_bytes(const lsa_dims& d, int64_t total_kept) {
    return (size_t)total_kept * d.H * (kDh + 2) * sizeof(float);
}

cudaError_t launch_small_step(const lsa_dims& d, const SeqTable& tab, const void* q_emb, const void* chunk_emb,
                              const void* q, const void* K, const void* V, int32_t* ids, float* out, float* lse,
                              float* part, uint32_t* ws, cudaStream_t stream) {
    int kmax = 0;
    for (int b = 0; b < d.B; ++b) kmax = std::max(kmax, tab.kept_off[b + 1] - tab.kept_off[b]);
    const float qscale = 1.4426950408889634f / sqrtf((float)kDh);
    const uint8_t *qe = (const uint8_t*)q_emb, *em = (const uint8_t*)chunk_emb, *q8 = (const uint8_t*)q;
    const uint8_t *K8 = (const uint8_t*)K, *V8 = (const uint8_t*)V;
    const bool cl = kmax <= kSmallMaxCluster;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)kmax;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kmax, d.H, d.B);
    cfg.blockDim = dim3(kSmallThreads, 1, 1);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = cl ? 1 : 0;
    const bool eb = d.emb_dtype == LSA_BF16, kb = d.kv_dtype == LSA_BF16;
#define LSA_SMALL_LAUNCH(E_, K_, C_)                                                                          \
    cudaLaunchKernelEx(&cfg, k_decode_small<E_, K_, C_>, qe, em, q8, K8, V8, ids, out, lse, part, tab, d.E, d.H, \
                       qscale, ws)
    if (cl) {
        if (eb && kb) return LSA_SMALL_LAUNCH(true, true, true);
        if (eb) return LSA_SMALL_LAUNCH(true, false, true);
        if (kb) return LSA_SMALL_LAUNCH(false, true, true);
        return LSA_SMALL_LAUNCH(false, false, true);
    }
    if (eb && kb) return LSA_SMALL_LAUNCH(true, true, false);
    if (eb) return LSA_SMALL_LAUNCH(true, false, false);
    if (kb) return LSA_SMALL_LAUNCH(false, true, false);
    return LSA_SMALL_LAUNCH(false, false, false);
#undef LSA_SMALL_LAUNCH
}

}  // namespace lsa
