// attention.cu - split-K flash-decode attention over the kept chunks only.
//
// FlashMemory-DeepSeek-V4 (review on dimensionstp.github.io, section 3-2 (3),
// steps 6-7): after the top-k keep mask, the decode step attends only over the
// kept chunks. For one decode query per sequence and head:
//     out = sum_t softmax_t(q . K_t / sqrt(Dh)) V_t    over the kept tokens t.
//
// Design (HBM-bound GEMV-like work: no tensor cores):
//  * The kept stages of all sequences form one global list (a stage is TOK
//    consecutive tokens of one kept chunk, all heads of a head slice). CTA c
//    of G takes stages [c*S/G, (c+1)*S/G): the split is balanced to one stage
//    whatever the batch or raggedness, and a CTA may cross sequence ends.
//  * One producer warp streams each stage's K and V rows straight from the full
//    cache through the kept chunk ids (or from a compact resident buffer) into a
//    3-deep shared-memory ring with 1-D bulk copies (TMA engine), completion on
//    mbarriers (transaction counts). No multicast; L2 evict-first hint.
//  * 8 consumer warps: LPH lanes per head hold 16 bytes of q and of the running
//    output each; dot products reduce with warp shuffles; online softmax in fp32
//    (log2 domain) over batches of 8 tokens; token groups split a stage when the
//    heads do not fill the 256 consumer threads.
//  * Each (CTA, sequence) pair writes an unnormalised partial (acc, m, l) to the
//    workspace; k_attn_merge combines a sequence's partials with the
//    log-sum-exp rule and writes out (and lse).
#include "lsa_device.cuh"

namespace lsa {

// Tunables (compile-time; the defaults are the measured best on B200).
#ifndef LSA_ATTN_WARPS
#define LSA_ATTN_WARPS 8        // consumer warps per CTA
#endif
#ifndef LSA_ATTN_STAGES
#define LSA_ATTN_STAGES 3       // ring slots
#endif
#ifndef LSA_ATTN_STAGE_BYTES
#define LSA_ATTN_STAGE_BYTES 32768  // bytes per operand (K or V) per ring slot
#endif

constexpr int kAttnConsumerWarps = LSA_ATTN_WARPS;
constexpr int kAttnConsumers = kAttnConsumerWarps * 32;
constexpr int kAttnThreads = kAttnConsumers + 32;
constexpr int kStageBytes = LSA_ATTN_STAGE_BYTES;
constexpr int kStages = LSA_ATTN_STAGES;
// Tokens each consumer group handles per stage when the stage is full-size: a
// stage holds kStageBytes / (HS*Dh*elem) tokens and a group covers LPH*HS threads,
// so TOK / TG = kStageBytes / (16 * consumers) for both element sizes.
constexpr int kTpgMax = kStageBytes / (16 * kAttnConsumers);
static_assert(kTpgMax >= 1 && (kTpgMax & (kTpgMax - 1)) == 0, "tokens per group must be a power of two");

struct AttnParams {
    int H;                // heads
    int HS;               // heads per CTA (head slice)
    int TG;               // token groups that hold tokens (<= consumers / (LPH * HS))
    int TOK;              // tokens per stage
    int SPC;              // stages per chunk (C / TOK)
    int G;                // CTAs per head slice
    int indexed;          // K/V read through chunk ids (1) or compact resident buffers (0)
    int64_t S;            // stages per head slice = sum k_b * SPC
    float qscale;         // log2(e) / sqrt(Dh)
    uint32_t row_bytes;   // bytes of one token's head slice = HS * Dh * elem
    uint64_t tok_stride;  // bytes of one token's full row = H * Dh * elem
};

size_t attn_smem_bytes(int lph) {
    return (size_t)2 * kStages * kStageBytes + (size_t)(kAttnConsumers / lph) * (kDh + 2) * 4 +
           (size_t)2 * kStages * 8;
}

__host__ __device__ __forceinline__ int64_t cta_of_stage(int64_t s, int64_t S, int G) {
    return ((s + 1) * G + S - 1) / S - 1;
}

template <bool BF16, int VEC>
__device__ __forceinline__ void unpack_vec(const uint4& v, float (&x)[VEC]) {
    if constexpr (BF16) {
        x[0] = bf16lo(v.x); x[1] = bf16hi(v.x); x[2] = bf16lo(v.y); x[3] = bf16hi(v.y);
        x[4] = bf16lo(v.z); x[5] = bf16hi(v.z); x[6] = bf16lo(v.w); x[7] = bf16hi(v.w);
    } else {
        x[0] = __uint_as_float(v.x); x[1] = __uint_as_float(v.y);
        x[2] = __uint_as_float(v.z); x[3] = __uint_as_float(v.w);
    }
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

// 2^x with the hardware approximation (relative error ~2^-22; 2^-inf = 0).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void consumer_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kAttnConsumers) : "memory");
}

// grid (G, H / HS), kAttnThreads threads, dynamic smem attn_smem_bytes(LPH).
// TPG: tokens per consumer group per stage (TOK / TG).
template <bool BF16, int TPG>
__global__ void __launch_bounds__(kAttnThreads, 1)
k_attn_split(const uint8_t* __restrict__ q, const uint8_t* __restrict__ K,
             const uint8_t* __restrict__ V, const int32_t* __restrict__ ids,
             float* __restrict__ part_o, float* __restrict__ part_ml, const SeqTable tab,
             const AttnParams ap, uint32_t* err, const int32_t* __restrict__ counts) {
    constexpr int ES = BF16 ? 2 : 4;
    constexpr int VEC = 16 / ES;   // head-dim elements per lane
    constexpr int LPH = kDh / VEC; // lanes per head
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t* sK = smem;
    uint8_t* sV = smem + kStages * kStageBytes;
    float* scratch = reinterpret_cast<float*>(smem + 2 * kStages * kStageBytes);
    uint64_t* bars = reinterpret_cast<uint64_t*>(scratch + (kAttnConsumers / LPH) * (kDh + 2));
    const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + kStages);
    __shared__ int s_abort;  // set by a consumer whose bounded wait gave up
    __shared__ int s_skip[kStages];  // ring slot holds no tokens (past the sequence's count, or a bad id)

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = blockIdx.x, hs = blockIdx.y;
    const int64_t s0 = (int64_t)c * ap.S / ap.G, s1 = (int64_t)(c + 1) * ap.S / ap.G;
    const uint32_t stage_bytes = (uint32_t)ap.TOK * ap.row_bytes;

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(full0 + 8 * i, 1);
            mbar_init(empty0 + 8 * i, kAttnConsumerWarps);
        }
        fence_mbar_init();
        s_abort = 0;
    }
    __syncthreads();
    pdl_trigger();

    if (warp == kAttnConsumerWarps) {
        // ------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            pdl_wait();  // chunk ids come from the preceding kernel
            int b = seq_of(tab.kept_off, tab.B, s0 / ap.SPC);
            for (int64_t s = s0, it = 0; s < s1; ++s, ++it) {
                const int slot = (int)(it % kStages);
                const uint32_t n = (uint32_t)(it / kStages);
                if (!mbar_wait(empty0 + 8 * slot, (n & 1u) ^ 1u, err)) break;
                const int64_t gidx = s / ap.SPC;
                const int64_t within = (s % ap.SPC) * ap.TOK;
                while (gidx >= tab.kept_off[b + 1]) ++b;
                if (counts != nullptr && gidx - tab.kept_off[b] >= (int64_t)counts[b]) {
                    s_skip[slot] = 1;                    // beyond this sequence's kept count
                    mbar_arrive(full0 + 8 * slot);       // release the slot without data
                    continue;
                }
                s_skip[slot] = 0;
                int64_t token0;
                if (ap.indexed) {
                    const int32_t id = ids[gidx];
                    const int n_b = tab.chunk_off[b + 1] - tab.chunk_off[b];
                    if (id < 0 || id >= n_b) {
                        set_error(err, kErrBadId);
                        s_skip[slot] = 1;               // the sequence attends over its valid ids only
                        mbar_arrive(full0 + 8 * slot);  // release the slot without data
                        continue;
                    }
                    token0 = ((int64_t)tab.chunk_off[b] + id) * tab.C + within;
                } else {
                    token0 = gidx * tab.C + within;
                }
                const uint32_t fb = full0 + 8 * slot;
                mbar_arrive_expect_tx(fb, 2 * stage_bytes);
                const uint8_t* ks = K + token0 * ap.tok_stride + (uint64_t)hs * ap.row_bytes;
                const uint8_t* vs = V + token0 * ap.tok_stride + (uint64_t)hs * ap.row_bytes;
                const uint32_t kd = smem_u32(sK + slot * kStageBytes);
                const uint32_t vd = smem_u32(sV + slot * kStageBytes);
                if (ap.HS == ap.H) {  // the stage is one contiguous run
                    bulk_g2s(kd, ks, stage_bytes, fb, pol);
                    bulk_g2s(vd, vs, stage_bytes, fb, pol);
                } else {              // one run per token
                    for (int t = 0; t < ap.TOK; ++t) {
                        bulk_g2s(kd + t * ap.row_bytes, ks + t * ap.tok_stride, ap.row_bytes, fb, pol);
                        bulk_g2s(vd + t * ap.row_bytes, vs + t * ap.tok_stride, ap.row_bytes, fb, pol);
                    }
                }
            }
        }
        return;
    }

    // ---------------------------------------------------- consumers
    const int li = tid % LPH;
    const int hl = (tid / LPH) % ap.HS;
    const int tg = tid / (LPH * ap.HS);
    const int h = hs * ap.HS + hl;
    const bool active = tg < ap.TG;  // warp-uniform: a warp holds whole groups or LPH = 32
    const uint32_t row = ap.row_bytes;
    const uint32_t lane_k = smem_u32(sK) + (uint32_t)(tg * TPG) * row + (uint32_t)hl * kDh * ES + li * 16;
    const uint32_t lane_v = lane_k + kStages * kStageBytes;

    int64_t it = 0;
    bool alive = true;
    int b = seq_of(tab.kept_off, tab.B, s0 / ap.SPC);
    for (int64_t seg0 = s0; seg0 < s1; ++b) {
        const int64_t seg1 = min(s1, (int64_t)tab.kept_off[b + 1] * ap.SPC);
        float qf[VEC];
        {
            const uint4 qv = *reinterpret_cast<const uint4*>(
                q + (((uint64_t)b * ap.H + h) * kDh) * ES + (uint64_t)li * 16);
            unpack_vec<BF16, VEC>(qv, qf);
#pragma unroll
            for (int e = 0; e < VEC; ++e) qf[e] *= ap.qscale;
        }
        float m = -INFINITY, l = 0.f, acc[VEC];
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] = 0.f;

        for (int64_t s = seg0; s < seg1; ++s, ++it) {
            const int slot = (int)(it % kStages);
            const uint32_t par = (uint32_t)(it / kStages) & 1u;
            if (!mbar_wait(full0 + 8 * slot, par, err)) {
                alive = false;
                s_abort = 1;
                break;
            }
            if (active && !*(volatile int*)&s_skip[slot]) {
                const uint32_t kb = lane_k + slot * kStageBytes;
                const uint32_t vb = lane_v + slot * kStageBytes;
                float sc[TPG];
#pragma unroll
                for (int j = 0; j < TPG; ++j) {
                    float x[VEC];
                    unpack_vec<BF16, VEC>(lds128(kb + j * row), x);
                    float d0 = 0.f, d1 = 0.f;
#pragma unroll
                    for (int e = 0; e < VEC; e += 2) {
                        d0 = fmaf(qf[e], x[e], d0);
                        d1 = fmaf(qf[e + 1], x[e + 1], d1);
                    }
                    sc[j] = d0 + d1;
                }
#pragma unroll
                for (int off = LPH / 2; off > 0; off >>= 1) {
#pragma unroll
                    for (int j = 0; j < TPG; ++j) sc[j] += __shfl_xor_sync(0xffffffffu, sc[j], off);
                }
                float mx = m;
#pragma unroll
                for (int j = 0; j < TPG; ++j) mx = fmaxf(mx, sc[j]);
                const float corr = ex2(m - mx);
                float p[TPG], psum = 0.f;
#pragma unroll
                for (int j = 0; j < TPG; ++j) {
                    p[j] = ex2(sc[j] - mx);
                    psum += p[j];
                }
                l = fmaf(l, corr, psum);
#pragma unroll
                for (int e = 0; e < VEC; ++e) acc[e] *= corr;
#pragma unroll
                for (int j = 0; j < TPG; ++j) {
                    float x[VEC];
                    unpack_vec<BF16, VEC>(lds128(vb + j * row), x);
#pragma unroll
                    for (int e = 0; e < VEC; ++e) acc[e] = fmaf(p[j], x[e], acc[e]);
                }
                m = mx;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty0 + 8 * slot);
        }

        // ---- combine the token groups of each head, then write this (CTA, sequence) partial
        const int64_t slot_id = (int64_t)c + b;
        float* po = part_o + ((uint64_t)slot_id * ap.H + h) * kDh + li * VEC;
        float* pml = part_ml + ((uint64_t)slot_id * ap.H + h) * 2;
        if (ap.TG == 1) {
            if (active) {
#pragma unroll
                for (int e = 0; e < VEC; e += 4)
                    *reinterpret_cast<float4*>(po + e) = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
                if (li == 0) {
                    pml[0] = m;
                    pml[1] = l;
                }
            }
        } else {
            if (active) {
                float* mine = scratch + (size_t)(tg * ap.HS + hl) * (kDh + 2);
#pragma unroll
                for (int e = 0; e < VEC; ++e) mine[li * VEC + e] = acc[e];
                if (li == 0) {
                    mine[kDh] = m;
                    mine[kDh + 1] = l;
                }
            }
            consumer_sync();
            if (tg == 0) {
                float M = -INFINITY;
                for (int g = 0; g < ap.TG; ++g) M = fmaxf(M, scratch[(size_t)(g * ap.HS + hl) * (kDh + 2) + kDh]);
                float L = 0.f, A[VEC];
#pragma unroll
                for (int e = 0; e < VEC; ++e) A[e] = 0.f;
                for (int g = 0; g < ap.TG; ++g) {
                    const float* o = scratch + (size_t)(g * ap.HS + hl) * (kDh + 2);
                    const float f = M == -INFINITY ? 0.f : ex2(o[kDh] - M);  // a group may hold no tokens
                    L = fmaf(o[kDh + 1], f, L);
#pragma unroll
                    for (int e = 0; e < VEC; ++e) A[e] = fmaf(o[li * VEC + e], f, A[e]);
                }
#pragma unroll
                for (int e = 0; e < VEC; e += 4)
                    *reinterpret_cast<float4*>(po + e) = make_float4(A[e], A[e + 1], A[e + 2], A[e + 3]);
                if (li == 0) {
                    pml[0] = M;
                    pml[1] = L;
                }
            }
        }
        seg0 = seg1;
        // every consumer passes the same barriers: leave together if any wait gave up
        consumer_sync();
        if (*(volatile int*)&s_abort) break;
    }
    (void)alive;
}

// Merge of the split partials of one (sequence, head) with the log-sum-exp rule.
// grid (B, H, kMergeDimSplit): a CTA merges kMergeDims of the Dh output columns over all of the
// sequence's slots. Warp g takes slots g, g + 8, ...; lane k owns column k of the CTA's 32. Each
// pass issues kMergeU slots' (m, l) and partial column together (one round trip) and folds them
// into the warp's running (m, l, acc); the eight warps are then combined in shared memory.
constexpr int kMergeDimSplit = 4;
constexpr int kMergeDims = kDh / kMergeDimSplit;          // 32 columns per CTA
constexpr int kMergeThreads = 256;
constexpr int kMergeGroups = kMergeThreads / kMergeDims;  // 8 slot groups (one warp each)
constexpr int kMergeU = 16;                               // slots in flight per thread
static_assert(kMergeDims == 32, "one lane per column");

__global__ void __launch_bounds__(kMergeThreads)
k_attn_merge(const float* __restrict__ part_o, const float* __restrict__ part_ml,
             float* __restrict__ out, float* __restrict__ lse, const SeqTable tab,
             const AttnParams ap) {
    __shared__ float s_m[kMergeGroups], s_l[kMergeGroups];
    __shared__ float s_acc[kMergeGroups][kMergeDims];
    const int b = blockIdx.x, h = blockIdx.y, tid = threadIdx.x, lane = tid & 31, g = tid >> 5;
    pdl_wait();
    const int64_t st0 = (int64_t)tab.kept_off[b] * ap.SPC;
    const int64_t st1 = (int64_t)tab.kept_off[b + 1] * ap.SPC - 1;
    const int c_lo = (int)cta_of_stage(st0, ap.S, ap.G);
    const int ns = (int)cta_of_stage(st1, ap.S, ap.G) - c_lo + 1;  // >= 1
    const uint64_t slot0 = (uint64_t)c_lo + b;
    const int d = blockIdx.z * kMergeDims + lane;
    const uint64_t sstride = (uint64_t)ap.H * kDh;
    const float* po = part_o + (slot0 * ap.H + h) * kDh + d;
    const float* pm = part_ml + (slot0 * ap.H + h) * 2;

    float m = -INFINITY, l = 0.f, a = 0.f;  // this warp's slots so far (m, l uniform in the warp)
    for (int i0 = g; i0 < ns; i0 += kMergeGroups * kMergeU) {
        float v[kMergeU], mu[kMergeU], lu[kMergeU];
#pragma unroll
        for (int u = 0; u < kMergeU; ++u) {  // past the last slot: reload it with no weight
            const int i = i0 + u * kMergeGroups;
            const int ic = i < ns ? i : ns - 1;
            v[u] = po[(uint64_t)ic * sstride];
            const float2 ml = *reinterpret_cast<const float2*>(pm + (uint64_t)ic * ap.H * 2);
            mu[u] = i < ns ? ml.x : -INFINITY;
            lu[u] = ml.y;
        }
        float mc = m;
#pragma unroll
        for (int u = 0; u < kMergeU; ++u) mc = fmaxf(mc, mu[u]);
        if (mc == -INFINITY) continue;  // no weight yet (slots of a count of 0)
        const float sc = m == -INFINITY ? 0.f : ex2(m - mc);
        l *= sc;
        a *= sc;
#pragma unroll
        for (int u = 0; u < kMergeU; ++u) {
            const float w = mu[u] == -INFINITY ? 0.f : ex2(mu[u] - mc);
            l = fmaf(w, lu[u], l);
            a = fmaf(w, v[u], a);
        }
        m = mc;
    }
    if (lane == 0) {
        s_m[g] = m;
        s_l[g] = l;
    }
    s_acc[g][lane] = a;
    __syncthreads();
    if (g != 0) return;
    float M = -INFINITY;
#pragma unroll
    for (int k = 0; k < kMergeGroups; ++k) M = fmaxf(M, s_m[k]);
    if (M == -INFINITY) {  // no kept token at all (a count of 0): empty output, lse = -inf
        out[((uint64_t)b * ap.H + h) * kDh + d] = 0.f;
        if (lse != nullptr && d == 0) lse[(uint64_t)b * ap.H + h] = -INFINITY;
        return;
    }
    float A = 0.f, L = 0.f;
#pragma unroll
    for (int k = 0; k < kMergeGroups; ++k) {
        const float w = s_m[k] == -INFINITY ? 0.f : ex2(s_m[k] - M);
        A = fmaf(w, s_acc[k][lane], A);
        L = fmaf(w, s_l[k], L);
    }
    out[((uint64_t)b * ap.H + h) * kDh + d] = A / L;
    if (lse != nullptr && d == 0) lse[(uint64_t)b * ap.H + h] = (M + log2f(L)) * 0.69314718055994531f;
}

// ------------------------------------------------------------------ host side
struct AttnLaunch {
    AttnParams ap;
    int slices;
    int lph;
    int tpg;  // tokens per consumer group per stage
    size_t smem;
};

template <bool BF16, int TPG>
cudaError_t set_split_attr(size_t smem) {
    return set_smem_attrs(k_attn_split<BF16, TPG>, (int)smem);
}

// Every (dtype, tokens-per-group) instantiation the planner can pick.
template <bool BF16>
cudaError_t set_split_attrs(size_t smem) {
    cudaError_t e = set_split_attr<BF16, 1>(smem);
    if (e == cudaSuccess && kTpgMax >= 2) e = set_split_attr<BF16, (kTpgMax >= 2 ? 2 : 1)>(smem);
    if (e == cudaSuccess && kTpgMax >= 4) e = set_split_attr<BF16, (kTpgMax >= 4 ? 4 : 1)>(smem);
    if (e == cudaSuccess && kTpgMax >= 8) e = set_split_attr<BF16, (kTpgMax >= 8 ? 8 : 1)>(smem);
    return e;
}

template <bool BF16>
cudaError_t launch_split(cudaLaunchConfig_t* cfg, int tpg, const void* q, const void* K, const void* V,
                         const int32_t* ids, float* part_o, float* part_ml, const SeqTable& tab,
                         const AttnParams& ap, uint32_t* err, const int32_t* counts) {
    const uint8_t *q8 = (const uint8_t*)q, *K8 = (const uint8_t*)K, *V8 = (const uint8_t*)V;
    switch (tpg) {
        case 1: return cudaLaunchKernelEx(cfg, k_attn_split<BF16, 1>, q8, K8, V8, ids, part_o, part_ml, tab, ap, err, counts);
        case 2: return cudaLaunchKernelEx(cfg, k_attn_split<BF16, (kTpgMax >= 2 ? 2 : 1)>, q8, K8, V8, ids, part_o, part_ml, tab, ap, err, counts);
        case 4: return cudaLaunchKernelEx(cfg, k_attn_split<BF16, (kTpgMax >= 4 ? 4 : 1)>, q8, K8, V8, ids, part_o, part_ml, tab, ap, err, counts);
        case 8: return cudaLaunchKernelEx(cfg, k_attn_split<BF16, (kTpgMax >= 8 ? 8 : 1)>, q8, K8, V8, ids, part_o, part_ml, tab, ap, err, counts);
    }
    return cudaErrorInvalidValue;
}

AttnLaunch plan_attention(const lsa_dims& d, const SeqTable& tab, int ctas_per_device, bool indexed) {
    AttnLaunch L = {};
    const int es = d.kv_dtype == LSA_BF16 ? 2 : 4;
    const int vec = 16 / es;
    L.lph = kDh / vec;
    AttnParams& ap = L.ap;
    ap.H = d.H;
    ap.HS = d.H < kAttnConsumers / L.lph ? d.H : kAttnConsumers / L.lph;
    const int groups = kAttnConsumers / (L.lph * ap.HS);
    L.slices = d.H / ap.HS;
    ap.row_bytes = (uint32_t)ap.HS * kDh * es;
    ap.tok_stride = (uint64_t)d.H * kDh * es;
    ap.TOK = kStageBytes / (int)ap.row_bytes;
    if (ap.TOK > d.chunk_len) ap.TOK = d.chunk_len;
    ap.TG = groups < ap.TOK ? groups : ap.TOK;  // groups beyond the stage's tokens stay idle
    L.tpg = ap.TOK / ap.TG;
    ap.SPC = d.chunk_len / ap.TOK;
    ap.S = (int64_t)tab.kept_off[d.B] * ap.SPC;
    int G = ctas_per_device / L.slices;
    if (G < 1) G = 1;
    if ((int64_t)G > ap.S) G = (int)ap.S;
    ap.G = G;
    ap.indexed = indexed ? 1 : 0;
    ap.qscale = 1.4426950408889634f / sqrtf((float)kDh);
    L.smem = attn_smem_bytes(L.lph);
    return L;
}

int attn_max_slots(int ctas_per_device, int B) { return ctas_per_device + B; }

cudaError_t attn_ctas_per_device(lsa_dtype kv, int num_sms, int* out) {
    int occ = 0;
    cudaError_t e = set_smem_attrs(k_attn_merge, 0);
    if (e != cudaSuccess) return e;
    if (kv == LSA_BF16) {
        e = set_split_attrs<true>(attn_smem_bytes(16));
        if (e != cudaSuccess) return e;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_attn_split<true, kTpgMax>, kAttnThreads,
                                                          attn_smem_bytes(16));
    } else {
        e = set_split_attrs<false>(attn_smem_bytes(32));
        if (e != cudaSuccess) return e;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_attn_split<false, kTpgMax>, kAttnThreads,
                                                          attn_smem_bytes(32));
    }
    if (e != cudaSuccess) return e;
    if (occ < 1) occ = 1;
    *out = occ * num_sms;
    return cudaSuccess;
}

cudaError_t launch_attention(const lsa_dims& d, const SeqTable& tab, int ctas_per_device,
                             const void* q, const void* K, const void* V, const int32_t* ids,
                             float* part_o, float* part_ml, float* out, float* lse, uint32_t* err,
                             cudaStream_t stream, bool pdl, const int32_t* counts) {
    const AttnLaunch L = plan_attention(d, tab, ctas_per_device, ids != nullptr);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;

    cudaLaunchConfig_t cfg = {};
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    cfg.gridDim = dim3(L.ap.G, L.slices, 1);
    cfg.blockDim = dim3(kAttnThreads, 1, 1);
    cfg.dynamicSmemBytes = L.smem;
    if (L.tpg != 1 && L.tpg != 2 && L.tpg != 4 && L.tpg != 8) return cudaErrorInvalidValue;
    cudaError_t e = d.kv_dtype == LSA_BF16
                        ? launch_split<true>(&cfg, L.tpg, q, K, V, ids, part_o, part_ml, tab, L.ap, err, counts)
                        : launch_split<false>(&cfg, L.tpg, q, K, V, ids, part_o, part_ml, tab, L.ap, err, counts);
    if (e != cudaSuccess) return e;

    cudaLaunchConfig_t mcfg = {};
    mcfg.stream = stream;
    mcfg.attrs = attr;
    mcfg.numAttrs = 1;  // the merge always follows the split kernel: overlap its launch
    mcfg.gridDim = dim3(d.B, d.H, kMergeDimSplit);
    mcfg.blockDim = dim3(kMergeThreads, 1, 1);
    mcfg.dynamicSmemBytes = 0;
    return cudaLaunchKernelEx(&mcfg, k_attn_merge, (const float*)part_o, (const float*)part_ml, out,
                              lse, tab, L.ap);
}

}  // namespace lsa
