// topk.cu - the top-k keep mask of Lookahead Sparse Attention.
//
// FlashMemory-DeepSeek-V4 (review on dimensionstp.github.io, section 3-2 (3),
// step 5): a top-k keep mask over the chunk scores decides which chunks stay
// resident. Ties go to the lower chunk index; -0.0 and +0.0 are equal.
//
// One CTA per sequence runs an exact radix select on order-preserving 32-bit
// keys (four 8-bit digit passes, most significant first) to find T, the k-th
// largest key, and how many keys equal to T must be kept. A final pass in index
// order keeps every key > T plus the lowest-index keys == T, and writes the kept
// indices in ascending order through a block-wide prefix count (ballots).
#include "lsa_device.cuh"

namespace lsa {

constexpr int kTopkThreads = 1024;
constexpr int kTopkWarps = kTopkThreads / 32;

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

// grid (B), 1024 threads. SMEM_KEYS: keys cached in dynamic smem (n_max * 4 bytes).
template <bool SMEM_KEYS>
__global__ void __launch_bounds__(kTopkThreads)
k_topk(const float* __restrict__ scores, int32_t* __restrict__ ids, const SeqTable tab,
       uint32_t* err) {
    extern __shared__ uint32_t skeys[];
    __shared__ uint32_t hist[256];
    __shared__ uint32_t s_prefix, s_need;
    __shared__ uint32_t w_gt[kTopkWarps], w_eq[kTopkWarps];
    __shared__ uint32_t o_gt[kTopkWarps], o_eq[kTopkWarps];
    __shared__ uint32_t t_gt, t_eq;

    const int b = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n = tab.chunk_off[b + 1] - tab.chunk_off[b];
    const int k = tab.kept_off[b + 1] - tab.kept_off[b];
    const float* s = scores + tab.chunk_off[b];
    int32_t* out = ids + tab.kept_off[b];

    pdl_wait();     // scores come from the preceding kernel
    pdl_trigger();

    bool bad = false;
    if constexpr (SMEM_KEYS) {
        for (int i = tid; i < n; i += kTopkThreads) skeys[i] = score_key(s[i], bad);
    } else {
        for (int i = tid; i < n; i += kTopkThreads) (void)score_key(s[i], bad);
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

    if (tid == 0) {
        s_prefix = 0;
        s_need = (uint32_t)k;
    }
    uint32_t prefix = 0, need = (uint32_t)k;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        const uint32_t himask = pass == 0 ? 0u : (0xFFFFFFFFu << (shift + 8));
        if (tid < 256) hist[tid] = 0;
        __syncthreads();
        for (int i0 = 0; i0 < n; i0 += kTopkThreads) {
            const int i = i0 + tid;
            uint32_t digit = 256;  // sentinel: not counted
            if (i < n) {
                const uint32_t key = key_at(i);
                if ((key & himask) == prefix) digit = (key >> shift) & 0xFFu;
            }
            // warp-aggregated histogram update: one atomic per distinct digit in the warp
            const uint32_t peers = __match_any_sync(0xffffffffu, digit);
            if (digit < 256 && (__ffs(peers) - 1) == lane) atomicAdd(&hist[digit], __popc(peers));
        }
        __syncthreads();
        if (warp == 0) {
            // lane l owns digits 255-8l .. 248-8l (descending)
            uint32_t h[8], sum = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                h[i] = hist[255 - 8 * lane - i];
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

    // ---- selection in index order
    const uint32_t lt_mask = (1u << lane) - 1u;
    uint32_t carry_gt = 0, carry_eq = 0;
    for (int i0 = 0; i0 < n; i0 += kTopkThreads) {
        const int i = i0 + tid;
        bool gt = false, eq = false;
        if (i < n) {
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
            if (pos < (uint32_t)k) out[pos] = i;
        } else if (eq && before_eq < need) {
            const uint32_t pos = before_gt + before_eq;
            if (pos < (uint32_t)k) out[pos] = i;
        }
        carry_gt += t_gt;
        carry_eq += t_eq;
        __syncthreads();
    }
}

constexpr size_t kTopkSmemKeyLimit = 200 * 1024;

// Raise the dynamic shared-memory limit of the top-k kernel (once per device).
cudaError_t topk_init_attrs() {
    return cudaFuncSetAttribute(k_topk<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kTopkSmemKeyLimit);
}

cudaError_t launch_topk(const lsa_dims& d, const SeqTable& tab, int max_n, const float* scores,
                        int32_t* ids, uint32_t* err, cudaStream_t stream, bool pdl) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    cfg.gridDim = dim3(d.B, 1, 1);
    cfg.blockDim = dim3(kTopkThreads, 1, 1);
    const size_t key_bytes = (size_t)max_n * 4;
    if (key_bytes <= kTopkSmemKeyLimit) {
        cfg.dynamicSmemBytes = key_bytes;
        return cudaLaunchKernelEx(&cfg, k_topk<true>, scores, ids, tab, err);
    }
    cfg.dynamicSmemBytes = 0;
    return cudaLaunchKernelEx(&cfg, k_topk<false>, scores, ids, tab, err);
}

}  // namespace lsa
