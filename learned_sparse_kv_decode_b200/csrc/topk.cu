// topk.cu - the top-k keep mask of Lookahead Sparse Attention.
//
// FlashMemory-DeepSeek-V4 (review on dimensionstp.github.io, section 3-2 (3),
// step 5): a top-k keep mask over the chunk scores decides which chunks stay
// resident. Ties go to the lower chunk index; -0.0 and +0.0 are equal.
//
// Exact radix select on order-preserving 32-bit keys, up to four 8-bit digit passes
// (most significant first), finding T, the k-th largest key, and how many keys
// equal to T must be kept. A final pass in index order keeps every key > T plus
// the lowest-index keys == T and writes the kept indices in ascending order. (The
// register kernel stops early when the bin holding the k-th key is kept whole.)
//
// One sequence runs on a thread-block cluster of CS CTAs (CS = 1..8): CTA r owns
// a contiguous slice of the sequence's keys. Each pass builds per-CTA digit
// histograms that are summed across the cluster through distributed shared memory
// (DSMEM); the ordered write uses per-CTA counts exchanged the same way. Cluster
// barriers are hardware barriers. Two kernels: k_topk_reg (keys in registers, up to
// 4096 per CTA: every workload here) and k_topk (keys in shared or global memory,
// for longer sequences).
#include "lsa_device.cuh"

namespace lsa {

constexpr int kTopkThreads = 1024;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkMaxCluster = 8;
constexpr int kTopkKeysPerCta = 2048;  // target slice size when choosing the cluster size
constexpr size_t kTopkSmemKeyLimit = 192 * 1024;

// Order-preserving map float -> uint32 (larger float -> larger key); -0 maps like +0.
// NaN maps to 0 (never preferred); NaN and +-Inf set `bad`.
__device__ __forceinline__ uint32_t score_key(float f, bool& bad) {
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7F800000u) == 0x7F800000u) {
        bad = true;
        if (u & 0x007FFFFFu) return 0u;
    }
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_size() {
    uint32_t n;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(n));
    return n;
}

// Load a u32 from the shared memory of CTA `rank` of this cluster at the same offset as `p`.
__device__ __forceinline__ uint32_t dsmem_ld(const uint32_t* p, uint32_t rank) {
    uint32_t remote, v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(p)), "r"(rank));
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(remote) : "memory");
    return v;
}

// Threshold keep mask (review section 3-2 (3), step 5: "top-k or threshold"): keep the
// chunks scoring at least tau, but no fewer than k_min (the fallback floor) and no more than
// the capacity k_b, always as a top-k set: k_eff = clamp(#{s >= tau}, min(k_min, k_b), k_b).
// counts[b] receives k_eff; id positions k_eff .. k_b-1 are set to -1.
struct ThresholdArgs {
    int enabled;
    float tau;
    int k_min;
    int32_t* counts;
};

// Sum of one value per thread over the CTA and then the cluster (every thread gets the total).
// `red` holds one slot per warp, `cta_total` one word that the cluster reads through DSMEM.
template <int WARPS>
__device__ __forceinline__ uint32_t cluster_sum(uint32_t v, uint32_t* red, uint32_t* cta_total, uint32_t cs) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = __reduce_add_sync(0xffffffffu, v);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    uint32_t t = 0;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) t += red[w];
    if (cs == 1) {
        __syncthreads();  // red is reused by the caller
        return t;
    }
    if (threadIdx.x == 0) *cta_total = t;
    cluster_sync_all();
    uint32_t parts[kTopkMaxCluster];
#pragma unroll
    for (int r = 0; r < kTopkMaxCluster; ++r) parts[r] = (uint32_t)r < cs ? dsmem_ld(cta_total, r) : 0u;
    uint32_t sum = 0;
#pragma unroll
    for (int r = 0; r < kTopkMaxCluster; ++r) sum += parts[r];
    cluster_sync_all();  // every CTA has read cta_total and red before they are reused
    return sum;
}

// grid (CS, B) with cluster (CS, 1, 1), 1024 threads.
// SMEM_KEYS: the CTA's key slice is cached in dynamic shared memory.
template <bool SMEM_KEYS>
__global__ void __launch_bounds__(kTopkThreads)
k_topk(const float* __restrict__ scores, int32_t* __restrict__ ids, const SeqTable tab,
       uint32_t* err, const ThresholdArgs th) {
    extern __shared__ uint32_t skeys[];
    __shared__ uint32_t hist[2][256];  // double-buffered: pass p uses hist[p & 1]
    __shared__ uint32_t tot[256];
    __shared__ uint32_t s_prefix, s_need;
    __shared__ uint32_t w_gt[kTopkWarps], w_eq[kTopkWarps];
    __shared__ uint32_t o_gt[kTopkWarps], o_eq[kTopkWarps];
    __shared__ uint32_t t_gt, t_eq;
    __shared__ uint32_t c_gt, c_eq;  // this CTA's totals of keys > T and == T (read by the cluster)
    __shared__ uint32_t s_red[kTopkWarps], s_cnt;

    const int b = blockIdx.y;
    const uint32_t rank = cluster_rank(), cs = cluster_size();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n = tab.chunk_off[b + 1] - tab.chunk_off[b];
    const int kcap = tab.kept_off[b + 1] - tab.kept_off[b];
    int k = kcap;
    const int slice = (n + (int)cs - 1) / (int)cs;
    const int lo = min(n, (int)rank * slice), hi = min(n, lo + slice);
    const int m = hi - lo;  // keys owned by this CTA: indices [lo, hi)
    const float* s = scores + tab.chunk_off[b] + lo;
    int32_t* out = ids + tab.kept_off[b];

    pdl_wait();     // scores come from the preceding kernel
    pdl_trigger();

    bool bad = false;
    if constexpr (SMEM_KEYS) {
        for (int i = tid; i < m; i += kTopkThreads) skeys[i] = score_key(s[i], bad);
    } else {
        for (int i = tid; i < m; i += kTopkThreads) (void)score_key(s[i], bad);
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) set_error(err, kErrNonFinite);

    auto key_at = [&](int i) -> uint32_t {
        if constexpr (SMEM_KEYS) {
            return skeys[i];
        } else {
            bool dummy = false;
            return score_key(__ldg(s + i), dummy);
        }
    };

    if (th.enabled) {
        bool dummy = false;
        const uint32_t tkey = score_key(th.tau, dummy);
        uint32_t c = 0;
        for (int i = tid; i < m; i += kTopkThreads) c += key_at(i) >= tkey;
        const int total = (int)cluster_sum<kTopkWarps>(c, s_red, &s_cnt, cs);
        k = max(min(total, kcap), min(th.k_min, kcap));
    }
    uint32_t prefix = 0, need = (uint32_t)k;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        const uint32_t himask = pass == 0 ? 0u : (0xFFFFFFFFu << (shift + 8));
        uint32_t* hp = hist[pass & 1];
        // hist[pass & 1] was last read two passes ago, before every CTA passed the previous
        // pass's cluster barrier, so it can be cleared now
        if (tid < 256) hp[tid] = 0;
        __syncthreads();
        for (int i0 = 0; i0 < m; i0 += kTopkThreads) {
            const int i = i0 + tid;
            uint32_t digit = 256;  // sentinel: not counted
            if (i < m) {
                const uint32_t key = key_at(i);
                if ((key & himask) == prefix) digit = (key >> shift) & 0xFFu;
            }
            // warp-aggregated histogram update: one atomic per distinct digit in the warp
            const uint32_t peers = __match_any_sync(0xffffffffu, digit);
            if (digit < 256 && (__ffs(peers) - 1) == lane) atomicAdd(&hp[digit], __popc(peers));
        }
        if (cs > 1) {
            cluster_sync_all();  // every CTA's histogram is complete and visible to the cluster
            if (tid < 256) {
                uint32_t v[kTopkMaxCluster];
#pragma unroll
                for (int r = 0; r < kTopkMaxCluster; ++r) v[r] = (uint32_t)r < cs ? dsmem_ld(&hp[tid], r) : 0u;
                uint32_t t = 0;
#pragma unroll
                for (int r = 0; r < kTopkMaxCluster; ++r) t += v[r];
                tot[tid] = t;
            }
        } else {
            __syncthreads();
            if (tid < 256) tot[tid] = hp[tid];
        }
        __syncthreads();
        if (warp == 0) {
            // lane l owns digits 255-8l .. 248-8l (descending)
            uint32_t h[8], sum = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                h[i] = tot[255 - 8 * lane - i];
                sum += h[i];
            }
            uint32_t incl = sum;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += v;
            }
            uint32_t above = incl - sum;  // keys with a larger digit
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (above < need && need <= above + h[i]) {
                    s_prefix = prefix | ((uint32_t)(255 - 8 * lane - i) << shift);
                    s_need = need - above;
                }
                above += h[i];
            }
        }
        __syncthreads();
        prefix = s_prefix;
        need = s_need;
    }
    const uint32_t T = prefix;  // the k-th largest key; keep `need` of the keys equal to T

    // ---- this CTA's counts of keys > T and == T, shared with the cluster
    {
        uint32_t g = 0, e = 0;
        for (int i = tid; i < m; i += kTopkThreads) {
            const uint32_t key = key_at(i);
            g += key > T;
            e += key == T;
        }
        g = __reduce_add_sync(0xffffffffu, g);
        e = __reduce_add_sync(0xffffffffu, e);
        if (lane == 0) {
            w_gt[warp] = g;
            w_eq[warp] = e;
        }
        __syncthreads();
        if (tid == 0) {
            uint32_t G = 0, E = 0;
            for (int w = 0; w < kTopkWarps; ++w) {
                G += w_gt[w];
                E += w_eq[w];
            }
            c_gt = G;
            c_eq = E;
        }
    }
    uint32_t carry_gt = 0, carry_eq = 0;  // keys > T and == T in lower-ranked CTAs
    if (cs > 1) {
        cluster_sync_all();
        uint32_t vg[kTopkMaxCluster], ve[kTopkMaxCluster];
#pragma unroll
        for (int r = 0; r < kTopkMaxCluster; ++r) {
            vg[r] = (uint32_t)r < rank ? dsmem_ld(&c_gt, r) : 0u;
            ve[r] = (uint32_t)r < rank ? dsmem_ld(&c_eq, r) : 0u;
        }
#pragma unroll
        for (int r = 0; r < kTopkMaxCluster; ++r) {
            carry_gt += vg[r];
            carry_eq += ve[r];
        }
    }

    // ---- selection in index order
    const uint32_t lt_mask = (1u << lane) - 1u;
    for (int i0 = 0; i0 < m; i0 += kTopkThreads) {
        const int i = i0 + tid;
        bool gt = false, eq = false;
        if (i < m) {
            const uint32_t key = key_at(i);
            gt = key > T;
            eq = key == T;
        }
        const uint32_t bg = __ballot_sync(0xffffffffu, gt), be = __ballot_sync(0xffffffffu, eq);
        if (lane == 0) {
            w_gt[warp] = __popc(bg);
            w_eq[warp] = __popc(be);
        }
        __syncthreads();
        if (warp == 0) {
            uint32_t g = w_gt[lane], e = w_eq[lane];
            uint32_t ig = g, ie = e;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const uint32_t vg = __shfl_up_sync(0xffffffffu, ig, off);
                const uint32_t ve = __shfl_up_sync(0xffffffffu, ie, off);
                if (lane >= off) {
                    ig += vg;
                    ie += ve;
                }
            }
            o_gt[lane] = ig - g;
            o_eq[lane] = ie - e;
            if (lane == 31) {
                t_gt = ig;
                t_eq = ie;
            }
        }
        __syncthreads();
        const uint32_t before_gt = carry_gt + o_gt[warp] + __popc(bg & lt_mask);
        const uint32_t before_eq = carry_eq + o_eq[warp] + __popc(be & lt_mask);
        // positions are < k by construction; the bound also guards the output buffer
        if (gt) {
            const uint32_t pos = before_gt + min(before_eq, need);
            if (pos < (uint32_t)k) out[pos] = lo + i;
        } else if (eq && before_eq < need) {
            const uint32_t pos = before_gt + before_eq;
            if (pos < (uint32_t)k) out[pos] = lo + i;
        }
        carry_gt += t_gt;
        carry_eq += t_eq;
        __syncthreads();
    }
    if (th.enabled) {
        for (int pos = k + (int)rank * kTopkThreads + tid; pos < kcap; pos += (int)cs * kTopkThreads) out[pos] = -1;
        if (rank == 0 && tid == 0) th.counts[b] = k;
    }
    if (cs > 1) cluster_sync_all();  // keep this CTA's shared memory alive until the cluster is done reading it
}

// ------------------------------------------------------------------ register-resident variant
// Each of the kTopkRegThreads threads keeps a contiguous run of R keys of its CTA's slice in
// registers, so each digit pass and the ordered write need one block barrier: the digit search
// runs redundantly in every warp and histograms are triple-buffered (the buffer a pass clears was
// last read two passes earlier). The keys arrive through a padded shared-memory transpose, so the
// global loads are coalesced while each thread still owns a contiguous run. The passes stop early
// once the bin holding the k-th key is kept whole (its count equals the keys still needed): the
// keep set is then every key >= the bin's lower edge, with no tie to break. The ordered write
// scans the two per-thread counts (kept outright, equal to T) packed into one word.
// In a cluster every exchange is a push: each CTA adds its histogram into every CTA's copy of
// the totals (remote red.add) and stores its counts into every CTA's table before the cluster
// barrier, so that after the barrier all reads are local and no CTA waits on a trailing barrier
// before it exits. The first barrier's arrive is issued before the loads and its wait after them.
#ifndef LSA_TOPK_HIST
#define LSA_TOPK_HIST 1  // histogram update: 0 = warp-aggregated (match.any), 1 = one atomic per key (faster)
#endif
#ifndef LSA_TOPK_REG_THREADS
#define LSA_TOPK_REG_THREADS 256
#endif
constexpr int kTopkRegThreads = LSA_TOPK_REG_THREADS;
constexpr int kTopkRegWarps = kTopkRegThreads / 32;

// Finds the digit d (of 256) where the keys above d number < need <= keys at or above d.
// Every lane of the calling warp returns the same (digit, keys above d, keys in bin d).
__device__ __forceinline__ void find_digit(const uint32_t* h256, uint32_t need, int lane,
                                           uint32_t& digit, uint32_t& above_out, uint32_t& bin_out) {
    uint32_t h[8], sum = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        h[i] = h256[255 - 8 * lane - i];
        sum += h[i];
    }
    uint32_t incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
    }
    uint32_t above = incl - sum;
    uint32_t found = 0xFFFFFFFFu, fa = 0, fb = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        if (found == 0xFFFFFFFFu && above < need && need <= above + h[i]) {
            found = (uint32_t)(255 - 8 * lane - i);
            fa = above;
            fb = h[i];
        }
        above += h[i];
    }
    const uint32_t who = __ballot_sync(0xffffffffu, found != 0xFFFFFFFFu);
    const int src = __ffs(who) - 1;  // exactly one lane holds the digit
    digit = __shfl_sync(0xffffffffu, found, src);
    above_out = __shfl_sync(0xffffffffu, fa, src);
    bin_out = __shfl_sync(0xffffffffu, fb, src);
}

// Add v to the u32 at the same shared-memory offset as `p` in CTA `rank` of this cluster.
__device__ __forceinline__ void dsmem_red_add(uint32_t* p, uint32_t rank, uint32_t v) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(p)), "r"(rank));
    asm volatile("red.relaxed.cluster.shared::cluster.add.u32 [%0], %1;" :: "r"(remote), "r"(v) : "memory");
}
// Store v to the u32 at the same shared-memory offset as `p` in CTA `rank` of this cluster.
__device__ __forceinline__ void dsmem_st(uint32_t* p, uint32_t rank, uint32_t v) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(p)), "r"(rank));
    asm volatile("st.shared::cluster.u32 [%0], %1;" :: "r"(remote), "r"(v) : "memory");
}
// The two halves of a cluster barrier, for work between the arrive and the wait.
__device__ __forceinline__ void cluster_arrive_release() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Shared-memory slot of slice index i in the load transpose: one pad word per 32 keeps both the
// coalesced writes (consecutive i) and the per-thread run reads (i = R * tid + j) conflict-free
// for R = 1, 2, 4, 8, 16.
__device__ __forceinline__ int topk_stage_slot(int i) { return i + (i >> 5); }

// grid (CS, B) with cluster (CS, 1, 1), kTopkRegThreads threads; a CTA's slice has at most
// kTopkRegThreads * R keys. Counts are packed 16 + 16 bits, so a sequence has at most 65535 keys.
template <int R>
__global__ void __launch_bounds__(kTopkRegThreads)
k_topk_reg(const float* __restrict__ scores, int32_t* __restrict__ ids, const SeqTable tab,
           uint32_t* err, const ThresholdArgs th) {
    constexpr int kSlice = kTopkRegThreads * R;
    __shared__ uint32_t hist[3][256];
    __shared__ uint32_t tot[2][256];  // cluster totals: every CTA adds its histogram into each CTA's copy
    __shared__ uint32_t stage[kSlice + kSlice / 32];
    __shared__ uint32_t r_cnt[kTopkMaxCluster];  // packed counts of each CTA, stored by that CTA
    __shared__ uint32_t w_cnt[kTopkRegWarps];
    __shared__ uint32_t s_red[kTopkRegWarps], s_cnt;

    const int b = blockIdx.y;
    const uint32_t rank = cluster_rank(), cs = cluster_size();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n = tab.chunk_off[b + 1] - tab.chunk_off[b];
    const int kcap = tab.kept_off[b + 1] - tab.kept_off[b];
    int k = kcap;
    const int slice = (n + (int)cs - 1) / (int)cs;
    const int lo = min(n, (int)rank * slice), hi = min(n, lo + slice);
    const int m = hi - lo;                     // keys of this CTA: [lo, hi)
    const int base = tid * R;                  // this thread's run: [base, base + R) within the slice
    const float* s = scores + tab.chunk_off[b] + lo;
    int32_t* out = ids + tab.kept_off[b];

    if (tid < 256) {
        hist[0][tid] = 0;
        hist[1][tid] = 0;
        tot[0][tid] = 0;
        tot[1][tid] = 0;
    }
    if (cs > 1) cluster_arrive_release();  // every CTA running, its totals zeroed (waited below)
    pdl_wait();  // scores come from the preceding kernel
    pdl_trigger();

    bool bad = false;
    {
        float v[R];  // every load in flight before the first store
#pragma unroll
        for (int j = 0; j < R; ++j) {
            const int i = j * kTopkRegThreads + tid;
            v[j] = i < m ? s[i] : 0.f;
        }
#pragma unroll
        for (int j = 0; j < R; ++j) {
            const int i = j * kTopkRegThreads + tid;
            stage[topk_stage_slot(i)] = i < m ? score_key(v[j], bad) : 0u;
        }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) set_error(err, kErrNonFinite);
    __syncthreads();
    uint32_t kr[R];
#pragma unroll
    for (int j = 0; j < R; ++j) kr[j] = stage[topk_stage_slot(base + j)];
    if (cs > 1) cluster_wait_acquire();

    if (th.enabled) {
        bool dummy = false;
        const uint32_t tkey = score_key(th.tau, dummy);
        uint32_t c = 0;
#pragma unroll
        for (int j = 0; j < R; ++j) c += (base + j < m && kr[j] >= tkey) ? 1u : 0u;
        const int total = (int)cluster_sum<kTopkRegWarps>(c, s_red, &s_cnt, cs);
        k = max(min(total, kcap), min(th.k_min, kcap));
    }
    // T = prefix: the k-th largest key, of which `need` are kept (lowest index first); with
    // `whole`, prefix is the lower edge of a bin kept whole and every key >= prefix is kept.
    uint32_t prefix = 0, need = (uint32_t)k;
    bool whole = false;
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
        if (whole) break;
        const int shift = 24 - 8 * pass;
        const uint32_t himask = pass == 0 ? 0u : (0xFFFFFFFFu << (shift + 8));
        uint32_t* hp = hist[pass % 3];
#pragma unroll
        for (int j = 0; j < R; ++j) {
            uint32_t digit = 256;
            if (base + j < m && (kr[j] & himask) == prefix) digit = (kr[j] >> shift) & 0xFFu;
#if LSA_TOPK_HIST == 0
            const uint32_t peers = __match_any_sync(0xffffffffu, digit);
            if (digit < 256 && (__ffs(peers) - 1) == lane) atomicAdd(&hp[digit], __popc(peers));
#else
            if (digit < 256) atomicAdd(&hp[digit], 1u);
#endif
        }
        if (tid < 256) hist[(pass + 1) % 3][tid] = 0;  // used next pass; last read two passes ago
        const uint32_t* h = hp;
        __syncthreads();
        if (cs > 1) {
            // tot[(pass + 1) % 2] was read last pass (every warp is past the barrier above); the
            // other CTAs add into it next pass, after the cluster barrier below
            if (tid < 256) {
                tot[(pass + 1) % 2][tid] = 0;
                const uint32_t v = hp[tid];
                if (v) {
                    for (uint32_t r = 0; r < cs; ++r) dsmem_red_add(&tot[pass % 2][tid], r, v);
                }
            }
            cluster_sync_all();
            h = tot[pass % 2];
        }
        uint32_t digit, above, inbin;
        find_digit(h, need, lane, digit, above, inbin);
        prefix |= digit << shift;
        need -= above;
        whole = need == inbin;  // the same decision in every thread of the cluster
    }
    // Kept outright: key >= T_lo, where T_lo = T + 1, or T itself when its bin is kept whole
    // (no key maps above +inf's 0xFF800000, so T + 1 does not wrap). Keys == T that are not kept
    // outright are tie candidates.
    const uint32_t T = prefix, T_lo = whole ? prefix : prefix + 1u;

    // ---- packed counts in index order: low half keys kept outright, high half tie candidates
    uint32_t c = 0;
#pragma unroll
    for (int j = 0; j < R; ++j) {
        if (base + j < m) c += kr[j] >= T_lo ? 1u : (kr[j] == T ? 0x10000u : 0u);
    }
    uint32_t ic = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, ic, off);
        if (lane >= off) ic += v;
    }
    if (lane == 31) w_cnt[warp] = ic;
    __syncthreads();
    uint32_t before = ic - c, cta = 0;
#pragma unroll
    for (int w = 0; w < kTopkRegWarps; ++w) {
        const uint32_t a = w_cnt[w];
        if (w < warp) before += a;
        cta += a;
    }
    if (cs > 1) {
        if ((uint32_t)tid < cs) dsmem_st(&r_cnt[rank], (uint32_t)tid, cta);
        cluster_sync_all();
#pragma unroll
        for (int r = 0; r < kTopkMaxCluster; ++r) before += (uint32_t)r < rank ? r_cnt[r] : 0u;
    }
    // ---- ordered write: every key kept outright, and the lowest-index `need` keys == T
    uint32_t before_g = before & 0xFFFFu, before_e = before >> 16;
#pragma unroll
    for (int j = 0; j < R; ++j) {
        if (base + j < m) {
            if (kr[j] >= T_lo) {
                const uint32_t pos = before_g + min(before_e, need);
                if (pos < (uint32_t)k) out[pos] = lo + base + j;
                ++before_g;
            } else if (kr[j] == T) {
                if (before_e < need) {
                    const uint32_t pos = before_g + before_e;
                    if (pos < (uint32_t)k) out[pos] = lo + base + j;
                }
                ++before_e;
            }
        }
    }
    if (th.enabled) {
        for (int pos = k + (int)rank * kTopkRegThreads + tid; pos < kcap; pos += (int)cs * kTopkRegThreads)
            out[pos] = -1;
        if (rank == 0 && tid == 0) th.counts[b] = k;
    }
}

// Raise the dynamic shared-memory limit of the top-k kernel (once per device).
cudaError_t topk_init_attrs() {
    cudaError_t e = set_smem_attrs(k_topk<true>, (int)kTopkSmemKeyLimit);
    if (e == cudaSuccess) e = set_smem_attrs(k_topk<false>, 0);
    if (e == cudaSuccess) e = set_smem_attrs(k_topk_reg<1>, 0);
    if (e == cudaSuccess) e = set_smem_attrs(k_topk_reg<2>, 0);
    if (e == cudaSuccess) e = set_smem_attrs(k_topk_reg<4>, 0);
    if (e == cudaSuccess) e = set_smem_attrs(k_topk_reg<8>, 0);
    if (e == cudaSuccess) e = set_smem_attrs(k_topk_reg<16>, 0);
    return e;
}

int topk_cluster_size(int max_n) {
    int cs = 1;
    while (cs < kTopkMaxCluster && cs * kTopkKeysPerCta < max_n) cs <<= 1;
    return cs;
}

cudaError_t launch_topk_impl(const lsa_dims& d, const SeqTable& tab, int max_n, const float* scores,
                             int32_t* ids, uint32_t* err, cudaStream_t stream, bool pdl, const ThresholdArgs& th) {
    const int cs = topk_cluster_size(max_n);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    cfg.gridDim = dim3(cs, d.B, 1);
    const int slice = (max_n + cs - 1) / cs;
    const int per_thread = (slice + kTopkRegThreads - 1) / kTopkRegThreads;
    if (per_thread <= 16) {
        cfg.blockDim = dim3(kTopkRegThreads, 1, 1);
        cfg.dynamicSmemBytes = 0;
        if (per_thread <= 1) return cudaLaunchKernelEx(&cfg, k_topk_reg<1>, scores, ids, tab, err, th);
        if (per_thread <= 2) return cudaLaunchKernelEx(&cfg, k_topk_reg<2>, scores, ids, tab, err, th);
        if (per_thread <= 4) return cudaLaunchKernelEx(&cfg, k_topk_reg<4>, scores, ids, tab, err, th);
        if (per_thread <= 8) return cudaLaunchKernelEx(&cfg, k_topk_reg<8>, scores, ids, tab, err, th);
        return cudaLaunchKernelEx(&cfg, k_topk_reg<16>, scores, ids, tab, err, th);
    }
    cfg.blockDim = dim3(kTopkThreads, 1, 1);
    const size_t key_bytes = (size_t)slice * 4;
    if (key_bytes <= kTopkSmemKeyLimit) {
        cfg.dynamicSmemBytes = key_bytes;
        return cudaLaunchKernelEx(&cfg, k_topk<true>, scores, ids, tab, err, th);
    }
    cfg.dynamicSmemBytes = 0;
    return cudaLaunchKernelEx(&cfg, k_topk<false>, scores, ids, tab, err, th);
}

cudaError_t launch_topk(const lsa_dims& d, const SeqTable& tab, int max_n, const float* scores,
                        int32_t* ids, uint32_t* err, cudaStream_t stream, bool pdl) {
    const ThresholdArgs none = {0, 0.f, 0, nullptr};
    return launch_topk_impl(d, tab, max_n, scores, ids, err, stream, pdl, none);
}

cudaError_t launch_threshold(const lsa_dims& d, const SeqTable& tab, int max_n, const float* scores,
                             float tau, int k_min, int32_t* ids, int32_t* counts, uint32_t* err,
                             cudaStream_t stream, bool pdl) {
    const ThresholdArgs th = {1, tau, k_min, counts};
    return launch_topk_impl(d, tab, max_n, scores, ids, err, stream, pdl, th);
}

}  // namespace lsa
