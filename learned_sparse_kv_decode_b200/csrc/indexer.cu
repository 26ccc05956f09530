// indexer.cu - the Neural Memory Indexer's score on FP8 compressed-K chunks.
//
// FlashMemory-DeepSeek-V4 (review on dimensionstp.github.io):
//  * section 3-2 (1): each compressed-K chunk is 132 bytes, 128 float8_e4m3 key values
//    followed by a float32 per-chunk dequant scale;
//  * section 3-2 (2): a chunk's relevance is s_i = sigmoid(sum_h ReLU(q_h . k_i) w_h) with
//    per-head queries q_h and fused head weights w_h; the released checkpoint has three
//    CSA layers whose scores are ensembled with a max or a mean;
//  * section 4-3: 128 heads, head dim 128.
// Queries arrive already quantised to e4m3 with a per-head dequant scale (the query-side
// projection, norm, RoPE and Hadamard transform are outside this library). Because both
// dequant scales are positive factors of the dot product, the kernel computes
//     v_il = sum_h w_lh * ReLU(ks_li * qs_blh * (q8_blh . k8_li)),  s_il = 1 / (1 + e^-v_il)
// and s_i = max_l s_il (or the mean).
//
// Per CTA: 128 chunks of one sequence. For each layer, the 128 x 132-byte rows arrive by one
// 1-D bulk copy (16-byte aligned window, a tail of < 16 bytes by plain loads) into a
// double-buffered raw tile and are re-laid out in shared memory into the fp8 keys (the
// no-swizzle K-major core-matrix layout) and the scales; the queries of all heads arrive by
// 2-D TMA tile loads into the same layout. The next layer loads while this one computes.
// One tcgen05 MMA chain of kind::f8f6f4
// (M = 128 chunks, N = heads, K = 128 in 4 steps of 32) accumulates q8 . k8 in TMEM
// (fp32); the epilogue reads a row per thread (tcgen05.ld) and applies scales, ReLU,
// head weights and the sigmoid.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "lsa_device.cuh"

namespace lsa {

constexpr int kIdxM = 128;      // chunks per CTA (MMA M)
constexpr int kIdxDim = 128;    // key / query dim (bytes of e4m3 per row)
constexpr int kIdxRowBytes = kIdxDim + 4;
constexpr int kIdxKChunks = kIdxDim / 16;  // 16-byte K-chunks per row

__device__ __forceinline__ uint64_t idx_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;  // descriptor version for sm_100; no swizzle, base offset 0
    return d;
}

// kind::f8f6f4 instruction descriptor: e4m3 A and B, fp32 D, both K-major, M x N.
__host__ __device__ constexpr uint32_t idx_idesc_e4m3_f32(int M, int N) {
    return (1u << 4)                         // D format: f32
           | (0u << 7)                       // A format: e4m3
           | (0u << 10)                      // B format: e4m3
           | ((uint32_t)(N >> 3) << 17)      // N / 8
           | ((uint32_t)(M >> 4) << 24);     // M / 16
}

__device__ __forceinline__ void idx_tma_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// Bytes of one raw tile buffer: up to 128 rows of 132 bytes plus 12 bytes of alignment slack.
constexpr int kIdxRawBytes = (kIdxM * kIdxRowBytes + 16 + 15) / 16 * 16;

// grid (ceil(maxN/128), B), 128 threads.
// dynamic smem: A keys [8 K-chunks][128 rows][16 B] | B queries [2][8][Hn][16 B] (double buffer)
//               | raw rows [2][kIdxRawBytes] (double buffer) | key scales [128] | query scales [Hn]
//               | head weights [Hn]
// ckv: compressed keys [L][sum N][132] (ckv_bytes long); tmQ: e4m3 queries [B*L*Hn rows][128],
// box 16 x Hn. Layer l+1's rows and queries load (1-D bulk copy + 2-D TMA) while layer l runs.
__global__ void __launch_bounds__(128)
k_score_fp8(const uint8_t* __restrict__ ckv, uint64_t ckv_bytes, const __grid_constant__ CUtensorMap tmQ,
            const float* __restrict__ q_scale, const float* __restrict__ head_w,
            float* __restrict__ scores, const SeqTable tab, int n_layers, int Hn, int mean,
            int64_t total_chunks, uint32_t tmem_cols, uint32_t* err) {
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ __align__(8) uint64_t load_bar[2];
    __shared__ __align__(8) uint64_t mma_bar;
    __shared__ uint32_t tmem_slot;

    const int b = blockIdx.y;
    const int n_b = tab.chunk_off[b + 1] - tab.chunk_off[b];
    const int r0 = blockIdx.x * kIdxM;
    pdl_trigger();
    if (r0 >= n_b) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rows = min(kIdxM, n_b - r0);

    const uint32_t qbytes = (uint32_t)Hn * kIdxDim;
    const uint32_t sA = smem_u32(smem);
    const uint32_t sB0 = sA + kIdxM * kIdxDim;
    uint8_t* raw0 = smem + kIdxM * kIdxDim + 2 * qbytes;
    float* ks = reinterpret_cast<float*>(raw0 + 2 * kIdxRawBytes);
    float* qs = ks + kIdxM;
    float* hw = qs + Hn;

    // byte window of layer l's rows: a 16-byte aligned bulk part plus a tail of < 16 bytes
    auto window = [&](int l, uint64_t& start_al, uint32_t& delta, uint32_t& bulk, uint32_t& tail) {
        const uint64_t off = ((uint64_t)l * total_chunks + (uint64_t)tab.chunk_off[b] + r0) * kIdxRowBytes;
        const uint64_t end = off + (uint64_t)rows * kIdxRowBytes;
        start_al = off & ~15ull;
        delta = (uint32_t)(off - start_al);
        uint64_t bulk_end = (end + 15) & ~15ull;
        const uint64_t cap = ckv_bytes & ~15ull;
        if (bulk_end > cap) bulk_end = cap;
        bulk = (uint32_t)(bulk_end - start_al);
        tail = (uint32_t)(end > bulk_end ? end - bulk_end : 0);
    };
    auto issue = [&](int l) {  // one thread: rows and queries of layer l into buffer l & 1
        const int buf = l & 1;
        uint64_t start_al;
        uint32_t delta, bulk, tail;
        window(l, start_al, delta, bulk, tail);
        const uint32_t bar = smem_u32(&load_bar[buf]);
        mbar_arrive_expect_tx(bar, bulk + qbytes);
        asm volatile(
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                smem_u32(raw0 + buf * kIdxRawBytes)),
            "l"(ckv + start_al), "r"(bulk), "r"(bar)
            : "memory");
        const int row = (b * n_layers + l) * Hn;
        const uint32_t sB = sB0 + buf * qbytes;
        for (int c = 0; c < kIdxKChunks; ++c) idx_tma_2d(sB + (uint32_t)c * Hn * 16, &tmQ, c * 16, row, bar);
    };

    if (tid == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmQ)) : "memory");
        mbar_init(smem_u32(&load_bar[0]), 1);
        mbar_init(smem_u32(&load_bar[1]), 1);
        mbar_init(smem_u32(&mma_bar), 1);
        fence_mbar_init();
        issue(0);
        if (n_layers > 1) issue(1);
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&tmem_slot)),
                     "r"(tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem_d = tmem_slot;
    const uint32_t idesc = idx_idesc_e4m3_f32(kIdxM, Hn);

    float combined = mean ? 0.f : -INFINITY;
    bool ok = true;
    for (int l = 0; l < n_layers; ++l) {
        const int buf = l & 1;
        uint8_t* raw = raw0 + buf * kIdxRawBytes;
        uint64_t start_al;
        uint32_t delta, bulk, tail;
        window(l, start_al, delta, bulk, tail);
        for (int h = tid; h < Hn; h += 128) {
            qs[h] = q_scale[((size_t)b * n_layers + l) * Hn + h];
            hw[h] = head_w[(size_t)l * Hn + h];
        }
        const bool landed = mbar_wait(smem_u32(&load_bar[buf]), (uint32_t)((l >> 1) & 1), err);
        if (tid < (int)(tail / 4))  // the last < 16 bytes of the tensor, past the aligned bulk part
            reinterpret_cast<uint32_t*>(raw + bulk)[tid] = __ldg(reinterpret_cast<const uint32_t*>(ckv + start_al + bulk) + tid);
        ok = __syncthreads_and(landed) != 0;
        if (!ok) break;
        // re-layout: row r's 128 key bytes -> 8 core-matrix rows of 16 bytes; its scale -> ks[r]
        {
            const int r = tid;
            const uint32_t* src = reinterpret_cast<const uint32_t*>(raw + delta) + r * (kIdxRowBytes / 4);
            uint32_t w[kIdxRowBytes / 4];
#pragma unroll
            for (int i = 0; i < kIdxRowBytes / 4; ++i) w[i] = r < rows ? src[i] : 0u;
#pragma unroll
            for (int c = 0; c < kIdxKChunks; ++c)
                *reinterpret_cast<uint4*>(smem + (c * kIdxM + r) * 16) =
                    make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
            ks[r] = __uint_as_float(w[kIdxDim / 4]);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // keys -> tensor core
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        __syncthreads();
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        if (tid == 0) {
            const uint32_t sB = sB0 + buf * qbytes;
            for (int ksx = 0; ksx < kIdxDim / 32; ++ksx) {
                // K-step ksx covers K-chunks 2ksx and 2ksx+1 (32 e4m3 values)
                const uint64_t ad = idx_desc(sA + (uint32_t)ksx * 2 * kIdxM * 16, kIdxM * 16, 128);
                const uint64_t bd = idx_desc(sB + (uint32_t)ksx * 2 * Hn * 16, (uint32_t)Hn * 16, 128);
                const uint32_t accum = ksx > 0 ? 1u : 0u;
                asm volatile(
                    "{\n\t.reg .pred p;\n\t"
                    "setp.ne.b32 p, %4, 0;\n\t"
                    "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
                    "l"(ad), "l"(bd), "r"(idesc), "r"(accum)
                    : "memory");
            }
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                             smem_u32(&mma_bar))
                         : "memory");
        }
        const bool done = mbar_wait(smem_u32(&mma_bar), (uint32_t)(l & 1), err);
        ok = __syncthreads_and(done) != 0;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        if (!ok) break;
        if (tid == 0 && l + 2 < n_layers) issue(l + 2);  // this buffer is free: prefetch two layers ahead

        // ---- epilogue: row 32*warp + lane; v = sum_h w_h ReLU(ks qs_h D[row][h]); sigmoid
        const float kscale = ks[warp * 32 + lane];
        float v = 0.f;
        const uint32_t taddr = tmem_d + ((uint32_t)(warp * 32) << 16);
        for (int c0 = 0; c0 < Hn; c0 += 16) {
            uint32_t r[16];
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                  "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
                  "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                : "r"(taddr + (uint32_t)c0));
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float a = kscale * qs[c0 + i] * __uint_as_float(r[i]);
                v = fmaf(hw[c0 + i], fmaxf(a, 0.f), v);
            }
        }
        const float s_l = 1.f / (1.f + expf(-v));
        combined = mean ? combined + s_l : fmaxf(combined, s_l);
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        __syncthreads();  // TMEM, keys and scales are reused by the next layer
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    }
    if (ok) {
        const int row = warp * 32 + lane;
        if (row < rows) scores[tab.chunk_off[b] + r0 + row] = mean ? combined / (float)n_layers : combined;
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_d), "r"(tmem_cols)
                     : "memory");
    }
}

size_t fp8_score_smem(int Hn) {
    return (size_t)kIdxM * kIdxDim + 2 * (size_t)Hn * kIdxDim + 2 * (size_t)kIdxRawBytes + (kIdxM + 2 * Hn) * 4;
}

cudaError_t fp8_init_attrs() { return set_smem_attrs(k_score_fp8, (int)fp8_score_smem(256)); }

cudaError_t make_tmap_u8_rows16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                                uint32_t box_rows) {
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (encode == nullptr) {
        cudaDriverEntryPointQueryResult q;
        void* fn = nullptr;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || fn == nullptr) return cudaErrorInvalidValue;
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols};
    const cuuint32_t box[2] = {16, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t launch_score_fp8(const lsa_dims& d, const SeqTable& tab, int max_n, int n_layers, int n_heads,
                             int mean, const uint8_t* ckv, const uint8_t* q8, const float* q_scale,
                             const float* head_w, float* scores, uint32_t* err, cudaStream_t stream,
                             bool pdl) {
    CUtensorMap tmQ;
    cudaError_t e = make_tmap_u8_rows16(&tmQ, q8, (uint64_t)d.B * n_layers * n_heads, kIdxDim, (uint32_t)n_heads);
    if (e != cudaSuccess) return e;
    uint32_t cols = 32;
    while ((int)cols < n_heads) cols <<= 1;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    cfg.gridDim = dim3((max_n + kIdxM - 1) / kIdxM, d.B, 1);
    cfg.blockDim = dim3(128, 1, 1);
    cfg.dynamicSmemBytes = fp8_score_smem(n_heads);
    const uint64_t ckv_bytes = (uint64_t)n_layers * (uint64_t)tab.chunk_off[d.B] * kIdxRowBytes;
    return cudaLaunchKernelEx(&cfg, k_score_fp8, ckv, ckv_bytes, tmQ, q_scale, head_w, scores, tab, n_layers, n_heads,
                              mean, (int64_t)tab.chunk_off[d.B], cols, err);
}

}  // namespace lsa
