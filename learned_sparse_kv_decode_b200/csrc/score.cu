// score.cu - chunk relevance scores of the Neural Memory Indexer.
//
// FlashMemory-DeepSeek-V4 (review on dimensionstp.github.io, section 3-2 (2);
// arXiv abstract): the indexer is a dual encoder, so a chunk's relevance is the
// inner product of the query-side embedding and the chunk-side embedding. With
// the ~64-token lookahead window (review, section 3-2 (3)) there are Q query
// embeddings per sequence and a chunk's score is the max over them (the same
// max the review gives for combining per-layer scores).
//
//   scores[i] = max_{j < Q} sum_e q_emb[b][j][e] * chunk_emb[i][e]      (fp32 accumulate)
//
// Kernels:
//  * k_score_bulk   - Q = 1, rows of at most 512 bytes: an HBM-bound stream over the
//    chunk embeddings staged into shared memory by 1-D bulk copies (TMA engine),
//    read back with 128-bit shared loads, the query piece held in registers, and a
//    warp shuffle reduction per row.
//  * k_score_stream - the other CUDA-core cases (Q > 1 without the tensor-core
//    path, longer rows): 128-bit streaming global loads, the queries in shared
//    memory.
//  * k_score_umma   - Q > 1 with bf16 embeddings: a tcgen05 tensor-core GEMM,
//    D[128 x Qp] = A[128 chunks x E] * B[Qp queries x E]^T accumulated in TMEM,
//    followed by a per-row max in the epilogue (tcgen05.ld).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "lsa_device.cuh"

namespace lsa {

// ============================================================== CUDA-core stream
template <bool BF16>
__device__ __forceinline__ void unpack16(const uint4& v, float (&x)[8]) {
    if constexpr (BF16) {
        x[0] = bf16lo(v.x); x[1] = bf16hi(v.x); x[2] = bf16lo(v.y); x[3] = bf16hi(v.y);
        x[4] = bf16lo(v.z); x[5] = bf16hi(v.z); x[6] = bf16lo(v.w); x[7] = bf16hi(v.w);
    } else {
        x[0] = __uint_as_float(v.x); x[1] = __uint_as_float(v.y);
        x[2] = __uint_as_float(v.z); x[3] = __uint_as_float(v.w);
    }
}

constexpr int kScoreThreads = 256;
constexpr int kScoreUnroll = 8;

// grid (row blocks, B); dynamic smem: Q*E floats (the queries of sequence b).
template <bool BF16>
__global__ void __launch_bounds__(kScoreThreads)
k_score_stream(const uint8_t* __restrict__ q_emb, const uint8_t* __restrict__ emb,
               float* __restrict__ scores, const SeqTable tab, int Q, int E, int rows_per_cta) {
    extern __shared__ float sq[];
    constexpr int ES = BF16 ? 2 : 4;
    constexpr int VEC = 16 / ES;  // elements per 16-byte piece
    const int b = blockIdx.y;
    const int n_b = tab.chunk_off[b + 1] - tab.chunk_off[b];
    const int r0 = blockIdx.x * rows_per_cta;
    pdl_trigger();
    if (r0 >= n_b) return;
    const int r1 = min(n_b, r0 + rows_per_cta);

    const size_t qbase = (size_t)b * Q * E;
    const int P = E / VEC;            // 16-byte pieces per row
    const int LPR = P < 32 ? P : 32;  // lanes per row
    const int RPW = 32 / LPR;         // rows per warp step
    const int PPL = P / LPR;          // pieces per lane
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane / LPR, li = lane % LPR;
    const int nwarps = blockDim.x >> 5;
    const size_t row_bytes = (size_t)E * ES;
    const uint8_t* base = emb + (size_t)tab.chunk_off[b] * row_bytes;
    float* out = scores + tab.chunk_off[b];
    const int step = nwarps * RPW;

    if (Q == 1 && PPL == 1) {
        // one query, one 16-byte piece per lane: the query piece lives in registers
        float qv[8];
        {
            const uint8_t* qp = q_emb + (qbase + (size_t)li * VEC) * ES;
            if constexpr (BF16) {
                unpack16<true>(*reinterpret_cast<const uint4*>(qp), qv);
            } else {
                const uint4 t = *reinterpret_cast<const uint4*>(qp);
                qv[0] = __uint_as_float(t.x); qv[1] = __uint_as_float(t.y);
                qv[2] = __uint_as_float(t.z); qv[3] = __uint_as_float(t.w);
            }
        }
        for (int wrow = r0 + warp * RPW; wrow < r1; wrow += step * kScoreUnroll) {
            const int row0 = wrow + sub;
            uint4 v[kScoreUnroll];
#pragma unroll
            for (int u = 0; u < kScoreUnroll; ++u) {
                const int row = row0 + u * step;
                v[u] = row < r1 ? ld_stream16(base + (size_t)row * row_bytes + (size_t)li * 16)
                                : make_uint4(0, 0, 0, 0);
            }
            float acc[kScoreUnroll];
#pragma unroll
            for (int u = 0; u < kScoreUnroll; ++u) {
                float x[8];
                unpack16<BF16>(v[u], x);
                acc[u] = 0.f;
#pragma unroll
                for (int e = 0; e < VEC; ++e) acc[u] = fmaf(qv[e], x[e], acc[u]);
                for (int off = LPR >> 1; off > 0; off >>= 1)
                    acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], off);
            }
            if (li == 0) {
#pragma unroll
                for (int u = 0; u < kScoreUnroll; ++u) {
                    const int row = row0 + u * step;
                    if (row < r1) out[row] = acc[u];
                }
            }
        }
        return;
    }

    for (int i = threadIdx.x; i < Q * E; i += blockDim.x) {
        if constexpr (BF16) {
            const uint16_t h = reinterpret_cast<const uint16_t*>(q_emb)[qbase + i];
            sq[i] = __uint_as_float((uint32_t)h << 16);
        } else {
            sq[i] = reinterpret_cast<const float*>(q_emb)[qbase + i];
        }
    }
    __syncthreads();

    // The loop bound is warp-uniform (every lane joins the shuffles); rows past r1 are masked.
    for (int wrow = r0 + warp * RPW; wrow < r1; wrow += step * kScoreUnroll) {
        const int row0 = wrow + sub;
        float best[kScoreUnroll];
#pragma unroll
        for (int u = 0; u < kScoreUnroll; ++u) best[u] = -INFINITY;
        for (int j = 0; j < Q; ++j) {
            float acc[kScoreUnroll];
#pragma unroll
            for (int u = 0; u < kScoreUnroll; ++u) acc[u] = 0.f;
            for (int p = 0; p < PPL; ++p) {
                const int piece = li + p * LPR;
                uint4 v[kScoreUnroll];
#pragma unroll
                for (int u = 0; u < kScoreUnroll; ++u) {
                    const int row = row0 + u * step;
                    v[u] = row < r1 ? ld_stream16(base + (size_t)row * row_bytes + (size_t)piece * 16)
                                    : make_uint4(0, 0, 0, 0);
                }
                const float* qp = sq + j * E + piece * VEC;
                float qv[8];
#pragma unroll
                for (int e = 0; e < VEC; ++e) qv[e] = qp[e];
#pragma unroll
                for (int u = 0; u < kScoreUnroll; ++u) {
                    float x[8];
                    unpack16<BF16>(v[u], x);
#pragma unroll
                    for (int e = 0; e < VEC; ++e) acc[u] = fmaf(qv[e], x[e], acc[u]);
                }
            }
#pragma unroll
            for (int u = 0; u < kScoreUnroll; ++u) {
                for (int off = LPR >> 1; off > 0; off >>= 1)
                    acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], off);
                best[u] = fmaxf(best[u], acc[u]);
            }
        }
        if (li == 0) {
#pragma unroll
            for (int u = 0; u < kScoreUnroll; ++u) {
                const int row = row0 + u * step;
                if (row < r1) out[row] = best[u];
            }
        }
    }
}

// ============================================================== TMA-staged stream (Q = 1)
// One CTA per slab of up to kScoreSlabBytes of consecutive rows of one sequence. Thread 0 issues
// the slab as kScoreStages 1-D bulk copies (TMA engine, L2 evict-first), each completing on its
// own mbarrier, all in flight at once. Once they have landed the warps read the rows back with
// 128-bit shared loads: P lanes per row (one 16-byte piece each) hold the query's matching piece
// in registers, kScoreUnroll rows at a time, and a shuffle reduction finishes each row. Rows of at most 512 bytes (every workload
// here); longer rows, and Q > 1 on the CUDA cores, take k_score_stream.
constexpr int kScoreStages = 4;
constexpr int kScoreSlabBytes = 32768;

template <bool BF16>
__global__ void __launch_bounds__(kScoreThreads)
k_score_bulk(const uint8_t* __restrict__ q_emb, const uint8_t* __restrict__ emb, float* __restrict__ scores,
             const SeqTable tab, int E, int rows_per_cta, uint32_t* err) {
    extern __shared__ __align__(128) uint8_t slab[];
    __shared__ __align__(8) uint64_t bars[kScoreStages];
    constexpr int ES = BF16 ? 2 : 4;
    constexpr int VEC = 16 / ES;
    const int b = blockIdx.y;
    const int n_b = tab.chunk_off[b + 1] - tab.chunk_off[b];
    const int r0 = blockIdx.x * rows_per_cta;
    pdl_trigger();
    if (r0 >= n_b) return;
    const int rows = min(n_b - r0, rows_per_cta);
    const uint32_t row_bytes = (uint32_t)E * ES;
    const int rps = (rows + kScoreStages - 1) / kScoreStages;  // rows per piece
    const uint32_t bar0 = smem_u32(bars);
    const uint32_t sbase = smem_u32(slab);
    if (threadIdx.x == 0) {
        for (int i = 0; i < kScoreStages; ++i) mbar_init(bar0 + 8 * i, 1);
        fence_mbar_init();
        const uint64_t pol = policy_evict_first();
        const uint8_t* src = emb + ((size_t)tab.chunk_off[b] + r0) * row_bytes;
        for (int i = 0; i < kScoreStages; ++i) {
            const int a = i * rps, e = min(rows, a + rps);
            if (a >= e) break;
            const uint32_t bytes = (uint32_t)(e - a) * row_bytes;
            mbar_arrive_expect_tx(bar0 + 8 * i, bytes);
            bulk_g2s(sbase + (uint32_t)a * row_bytes, src + (size_t)a * row_bytes, bytes, bar0 + 8 * i, pol);
        }
    }

    const int P = E / VEC;  // 16-byte pieces per row (<= 32)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int RPW = 32 / P;  // rows per warp step
    const int sub = lane / P, li = lane % P;
    const int step = (kScoreThreads / 32) * RPW;
    float qv[8];
    {
        const uint8_t* qp = q_emb + ((size_t)b * E + (size_t)li * VEC) * ES;
        const uint4 t = *reinterpret_cast<const uint4*>(qp);
        float x[8];
        unpack16<BF16>(t, x);
#pragma unroll
        for (int e = 0; e < 8; ++e) qv[e] = x[e];
    }
    __syncthreads();  // the barriers are initialised before anyone waits on them
    // every piece is waited for (bounded), even after a wait gave up: no copy is in flight at exit
    bool ok = true;
    for (int i = 0; i < kScoreStages && i * rps < rows; ++i) {
        const bool landed = mbar_wait(bar0 + 8 * i, 0u, err);
        ok = ok && landed;
    }
    float* out = scores + tab.chunk_off[b] + r0;
    // kScoreUnroll rows per warp and iteration, independent until their stores; the loop bound is
    // warp-uniform (every lane joins the shuffles) and rows past the slab are masked
    for (int wrow = warp * RPW; wrow < rows; wrow += step * kScoreUnroll) {
        const int row0 = wrow + sub;
        float acc[kScoreUnroll];
#pragma unroll
        for (int u = 0; u < kScoreUnroll; ++u) {
            const int row = row0 + u * step;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (row < rows && ok)
                asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                             : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                             : "r"(sbase + (uint32_t)row * row_bytes + (uint32_t)li * 16));
            float x[8];
            unpack16<BF16>(v, x);
            acc[u] = 0.f;
#pragma unroll
            for (int e = 0; e < VEC; ++e) acc[u] = fmaf(qv[e], x[e], acc[u]);
        }
#pragma unroll
        for (int u = 0; u < kScoreUnroll; ++u)
            for (int off = P >> 1; off > 0; off >>= 1) acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], off);
        if (li == 0 && ok) {
#pragma unroll
            for (int u = 0; u < kScoreUnroll; ++u) {
                const int row = row0 + u * step;
                if (row < rows) out[row] = acc[u];
            }
        }
    }
}

// ============================================================== tcgen05 GEMM + row max
// Shared-memory operand layout: K-major, no swizzle ("interleaved" canonical layout),
// written directly by 2-D TMA tile loads. The tile of K-chunk c (8 bf16 = 16 bytes of
// every row) is one box of [rows x 16 bytes], stored rows-contiguous, so an 8-row x
// 16-byte core matrix is 128 contiguous bytes, 8-row groups are SBO = 128 bytes apart
// and K-chunks are LBO = rows * 16 bytes apart.
__device__ __forceinline__ uint64_t umma_desc_k_noswizzle(uint32_t saddr, uint32_t lbo,
                                                          uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;  // descriptor version for sm_100
    // base offset 0, absolute LBO mode off, layout type 0 = no swizzle
    return d;
}

// Instruction descriptor of kind::f16: bf16 A and B, fp32 D, both K-major, M x N.
__host__ __device__ constexpr uint32_t umma_idesc_bf16_f32(int M, int N) {
    return (1u << 4)                         // D format: f32
           | (1u << 7)                       // A format: bf16
           | (1u << 10)                      // B format: bf16
           | ((uint32_t)(N >> 3) << 17)      // N / 8
           | ((uint32_t)(M >> 4) << 24);     // M / 16
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 2-D TMA tile load (no multicast) of the box at (x = column, y = row) into shared memory.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

constexpr int kUmmaM = 128;

// grid (ceil(maxN/128), B), 128 threads; dynamic smem: A (128*E*2) + B (Np*E*2), 1 KiB aligned.
// tmA: chunk embeddings [sum N][E] bf16, box 8 x 128; tmB: query embeddings [B*Q][E], box 8 x Np.
__global__ void __launch_bounds__(128)
k_score_umma(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
             float* __restrict__ scores, const SeqTable tab, int Q, int Np, int E,
             uint32_t tmem_cols, uint32_t* err) {
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ __align__(8) uint64_t load_bar;
    __shared__ __align__(8) uint64_t mma_bar;
    __shared__ uint32_t tmem_slot;

    const int b = blockIdx.y;
    const int n_b = tab.chunk_off[b + 1] - tab.chunk_off[b];
    const int r0 = blockIdx.x * kUmmaM;
    pdl_trigger();
    if (r0 >= n_b) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int KC = E / 8;  // 16-byte K-chunks per row
    const uint32_t sA = smem_u32(smem), sB = sA + (uint32_t)kUmmaM * E * 2;

    if (tid == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
        mbar_init(smem_u32(&load_bar), 1);
        mbar_init(smem_u32(&mma_bar), 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&tmem_slot)),
                     "r"(tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_d = tmem_slot;

    bool loaded = true;
    if (tid == 0) {
        // one thread stages both operands; rows past the tensor read as zeros, rows of the next
        // sequence (inside the tensor) are loaded and masked in the epilogue
        const uint32_t lb = smem_u32(&load_bar);
        mbar_arrive_expect_tx(lb, (uint32_t)(kUmmaM + Np) * E * 2);
        const int rowA = tab.chunk_off[b] + r0, rowB = b * Q;
        for (int c = 0; c < KC; ++c) {
            tma_load_2d(sA + (uint32_t)c * kUmmaM * 16, &tmA, c * 8, rowA, lb);
            tma_load_2d(sB + (uint32_t)c * Np * 16, &tmB, c * 8, rowB, lb);
        }
        loaded = mbar_wait(lb, 0, err);
        if (loaded) {
            const uint32_t idesc = umma_idesc_bf16_f32(kUmmaM, Np);
            for (int ks = 0; ks < E / 16; ++ks) {
                // K-step ks covers K-chunks 2ks and 2ks+1
                const uint64_t ad = umma_desc_k_noswizzle(sA + (uint32_t)ks * 2 * kUmmaM * 16, kUmmaM * 16, 128);
                const uint64_t bd = umma_desc_k_noswizzle(sB + (uint32_t)ks * 2 * Np * 16, (uint32_t)Np * 16, 128);
                const uint32_t accum = ks > 0 ? 1u : 0u;
                asm volatile(
                    "{\n\t.reg .pred p;\n\t"
                    "setp.ne.b32 p, %4, 0;\n\t"
                    "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
                    "l"(ad), "l"(bd), "r"(idesc), "r"(accum)
                    : "memory");
            }
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                             smem_u32(&mma_bar))
                         : "memory");
        } else {
            mbar_arrive(smem_u32(&mma_bar));  // no MMA was issued: release the waiters
        }
    }
    // warp-uniform: the tcgen05.ld below is .sync.aligned
    const bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&mma_bar), 0, err) && loaded);
    const bool all_ok = __syncthreads_and(ok);
    tc_fence_after();

    // ---- epilogue: row r0 + 32*warp + lane lives in TMEM lane 32*warp + lane
    float best = -INFINITY;
    if (all_ok) {
        const uint32_t taddr = tmem_d + ((uint32_t)(warp * 32) << 16);
        for (int c0 = 0; c0 < Np; c0 += 16) {
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
            for (int i = 0; i < 16; ++i)
                if (c0 + i < Q) best = fmaxf(best, __uint_as_float(r[i]));
        }
        const int row = r0 + warp * 32 + lane;
        if (row < n_b) scores[tab.chunk_off[b] + row] = best;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_d),
                     "r"(tmem_cols)
                     : "memory");
    }
}

// Shared-memory descriptor of a K-major operand in the 128-byte-swizzled layout (sm_100 layout
// type 2): rows of 128 bytes (64 bf16), 8-row atoms of 1 KiB (SBO = 1024); LBO unused (1).
__device__ __forceinline__ uint64_t umma_desc_k_sw128(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// The same GEMM + row max with 128-byte-swizzled operand tiles, for E a multiple of 64 (<= 256).
// The E dimension is split into E/64 regions of 64 columns; one TMA box per region and operand
// (box [64 x 128 rows] for the chunks, [64 x Np] for the queries) lands in 128-byte rows, and
// each region has its own mbarrier so the MMAs of region r start while later regions land.
// grid (ceil(maxN/128), B), 128 threads; dynamic smem: E/64 * (128 + Np) * 128 B + 1 KiB.
constexpr int kScoreSwRegionsMax = 4;
__global__ void __launch_bounds__(128)
k_score_umma_sw(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                float* __restrict__ scores, const SeqTable tab, int Q, int Np, int E, uint32_t tmem_cols,
                uint32_t* err) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t load_bar[kScoreSwRegionsMax];
    __shared__ __align__(8) uint64_t mma_bar;
    __shared__ uint32_t tmem_slot;

    const int b = blockIdx.y;
    const int n_b = tab.chunk_off[b + 1] - tab.chunk_off[b];
    const int r0 = blockIdx.x * kUmmaM;
    pdl_trigger();
    if (r0 >= n_b) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int R = E / 64;  // regions of 64 columns
    const uint32_t sA = (smem_u32(smem_raw) + 1023u) & ~1023u;  // swizzle atoms need 1 KiB alignment
    const uint32_t sB = sA + (uint32_t)R * kUmmaM * 128;

    if (tid == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
        for (int r = 0; r < R; ++r) mbar_init(smem_u32(&load_bar[r]), 1);
        mbar_init(smem_u32(&mma_bar), 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&tmem_slot)),
                     "r"(tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_d = tmem_slot;

    bool loaded = true;
    if (tid == 0) {
        // rows past the tensor read as zeros; rows of the next sequence are loaded and masked
        pdl_wait();
        const int rowA = tab.chunk_off[b] + r0, rowB = b * Q;
        for (int r = 0; r < R; ++r) {
            const uint32_t lb = smem_u32(&load_bar[r]);
            mbar_arrive_expect_tx(lb, (uint32_t)(kUmmaM + Np) * 128);
            tma_load_2d(sA + (uint32_t)r * kUmmaM * 128, &tmA, 64 * r, rowA, lb);
            tma_load_2d(sB + (uint32_t)r * Np * 128, &tmB, 64 * r, rowB, lb);
        }
        const uint32_t idesc = umma_idesc_bf16_f32(kUmmaM, Np);
        for (int r = 0; r < R && loaded; ++r) {
            loaded = mbar_wait(smem_u32(&load_bar[r]), 0, err);
            if (!loaded) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {  // 16 columns (32 bytes) per MMA K-step
                const uint64_t ad = umma_desc_k_sw128(sA + (uint32_t)r * kUmmaM * 128 + (uint32_t)kk * 32);
                const uint64_t bd = umma_desc_k_sw128(sB + (uint32_t)r * Np * 128 + (uint32_t)kk * 32);
                const uint32_t accum = (r > 0 || kk > 0) ? 1u : 0u;
                asm volatile(
                    "{\n\t.reg .pred p;\n\t"
                    "setp.ne.b32 p, %4, 0;\n\t"
                    "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
                    "l"(ad), "l"(bd), "r"(idesc), "r"(accum)
                    : "memory");
            }
        }
        if (loaded) {
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                             smem_u32(&mma_bar))
                         : "memory");
        } else {
            // a load gave up: wait (bounded) for every copy issued, then release the waiters
            for (int r = 0; r < R; ++r) mbar_wait(smem_u32(&load_bar[r]), 0, err);
            mbar_arrive(smem_u32(&mma_bar));
        }
    }
    const bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&mma_bar), 0, err) && loaded);
    const bool all_ok = __syncthreads_and(ok);
    tc_fence_after();

    // ---- epilogue: row r0 + 32*warp + lane lives in TMEM lane 32*warp + lane
    float best = -INFINITY;
    if (all_ok) {
        const uint32_t taddr = tmem_d + ((uint32_t)(warp * 32) << 16);
        for (int c0 = 0; c0 < Np; c0 += 16) {
            uint32_t rr[16];
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                : "=r"(rr[0]), "=r"(rr[1]), "=r"(rr[2]), "=r"(rr[3]), "=r"(rr[4]), "=r"(rr[5]),
                  "=r"(rr[6]), "=r"(rr[7]), "=r"(rr[8]), "=r"(rr[9]), "=r"(rr[10]), "=r"(rr[11]),
                  "=r"(rr[12]), "=r"(rr[13]), "=r"(rr[14]), "=r"(rr[15])
                : "r"(taddr + (uint32_t)c0));
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
            for (int i = 0; i < 16; ++i)
                if (c0 + i < Q) best = fmaxf(best, __uint_as_float(rr[i]));
        }
        const int row = r0 + warp * 32 + lane;
        if (row < n_b) scores[tab.chunk_off[b] + row] = best;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_d),
                     "r"(tmem_cols)
                     : "memory");
    }
}

// Host: a 2-D tensor map over a row-major bf16 matrix [rows][cols], box [64 columns x box_rows],
// 128-byte swizzle, zero fill outside the tensor (cols a multiple of 64).
cudaError_t make_tmap_sw128(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows);

// Host: a 2-D tensor map over a row-major bf16 matrix [rows][cols] with a box of
// [box_rows x 8 columns] (16 bytes per row), no swizzle, zero fill outside the tensor.
cudaError_t make_tmap_rows16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
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
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {8, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_tmap_sw128(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (encode == nullptr) {
        cudaDriverEntryPointQueryResult q;
        void* fn = nullptr;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || fn == nullptr) return cudaErrorInvalidValue;
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// ============================================================== launchers
// Raise the dynamic shared-memory limit of the score kernels (once per device).
// The limits are the largest requests the launchers make (E <= 256 and Q <= 256 for the
// tensor-core kernel; Q*E*4 <= 200 KiB for the stream kernel, checked on the host).
constexpr int kScoreStreamSmemMax = 200 * 1024;
size_t score_umma_smem(int E, int Np);
size_t score_umma_sw_smem(int E, int Np);
cudaError_t score_init_attrs() {
    cudaError_t e = set_smem_attrs(k_score_umma, (int)score_umma_smem(256, 256));
    if (e == cudaSuccess) e = set_smem_attrs(k_score_umma_sw, (int)score_umma_sw_smem(256, 256));
    if (e == cudaSuccess) e = set_smem_attrs(k_score_stream<true>, kScoreStreamSmemMax);
    if (e == cudaSuccess) e = set_smem_attrs(k_score_stream<false>, kScoreStreamSmemMax);
    if (e == cudaSuccess) e = set_smem_attrs(k_score_bulk<true>, kScoreSlabBytes);
    if (e == cudaSuccess) e = set_smem_attrs(k_score_bulk<false>, kScoreSlabBytes);
    return e;
}

// A and B tiles plus 4 KiB of slack after them (never read when the descriptors are right).
size_t score_umma_smem(int E, int Np) { return (size_t)(kUmmaM + Np) * E * 2 + 4096; }
// E/64 regions of (128 + Np) rows x 128 B, plus 1 KiB to align the swizzle atoms.
size_t score_umma_sw_smem(int E, int Np) { return (size_t)(E / 64) * (kUmmaM + Np) * 128 + 1024; }

bool score_uses_umma(const lsa_dims& d) {
    return d.Q > 1 && d.emb_dtype == LSA_BF16 && d.E % 16 == 0 && d.E <= 256 && d.Q <= 256;
}

cudaError_t launch_score(const lsa_dims& d, const SeqTable& tab, int max_n, const void* q_emb,
                         const void* chunk_emb, float* scores, uint32_t* err, int num_sms,
                         cudaStream_t stream, bool pdl) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;

    if (score_uses_umma(d)) {
        const int Np = (d.Q + 15) / 16 * 16;
        uint32_t cols = 32;
        while ((int)cols < Np) cols <<= 1;
        CUtensorMap tmA, tmB;
        cfg.gridDim = dim3((max_n + kUmmaM - 1) / kUmmaM, d.B, 1);
        cfg.blockDim = dim3(128, 1, 1);
        if (d.E % 64 == 0) {  // 128-byte rows: one TMA box per 64-column region and operand
            cudaError_t e = make_tmap_sw128(&tmA, chunk_emb, (uint64_t)tab.chunk_off[d.B], d.E, kUmmaM);
            if (e == cudaSuccess) e = make_tmap_sw128(&tmB, q_emb, (uint64_t)d.B * d.Q, d.E, (uint32_t)Np);
            if (e != cudaSuccess) return e;
            cfg.dynamicSmemBytes = score_umma_sw_smem(d.E, Np);
            return cudaLaunchKernelEx(&cfg, k_score_umma_sw, tmA, tmB, scores, tab, d.Q, Np, d.E, cols, err);
        }
        cudaError_t e = make_tmap_rows16(&tmA, chunk_emb, (uint64_t)tab.chunk_off[d.B], d.E, kUmmaM);
        if (e == cudaSuccess) e = make_tmap_rows16(&tmB, q_emb, (uint64_t)d.B * d.Q, d.E, (uint32_t)Np);
        if (e != cudaSuccess) return e;
        cfg.gridDim = dim3((max_n + kUmmaM - 1) / kUmmaM, d.B, 1);
        cfg.blockDim = dim3(128, 1, 1);
        cfg.dynamicSmemBytes = score_umma_smem(d.E, Np);
        return cudaLaunchKernelEx(&cfg, k_score_umma, tmA, tmB, scores, tab, d.Q, Np, d.E, cols, err);
    }
    const int es = d.emb_dtype == LSA_BF16 ? 2 : 4;
    const int P = d.E * es / 16;
    if (d.Q == 1 && P <= 32) {
        // TMA-staged slabs of at most kScoreSlabBytes, at least two per SM when the rows allow
        const int row_bytes = d.E * es;
        const int total_rows = tab.chunk_off[d.B];
        int rpc = kScoreSlabBytes / row_bytes;
        const int spread = (total_rows + 2 * num_sms - 1) / (2 * num_sms);
        if (spread < rpc) rpc = spread;
        if (rpc < 1) rpc = 1;
        cfg.gridDim = dim3((max_n + rpc - 1) / rpc, d.B, 1);
        cfg.blockDim = dim3(kScoreThreads, 1, 1);
        cfg.dynamicSmemBytes = (size_t)rpc * row_bytes;
        if (d.emb_dtype == LSA_BF16)
            return cudaLaunchKernelEx(&cfg, k_score_bulk<true>, (const uint8_t*)q_emb, (const uint8_t*)chunk_emb,
                                      scores, tab, d.E, rpc, err);
        return cudaLaunchKernelEx(&cfg, k_score_bulk<false>, (const uint8_t*)q_emb, (const uint8_t*)chunk_emb,
                                  scores, tab, d.E, rpc, err);
    }
    const int LPR = P < 32 ? P : 32;
    const int rows_step = (kScoreThreads / 32) * (32 / LPR) * kScoreUnroll;
    int total_rows = tab.chunk_off[d.B];
    int want = (total_rows + 4 * num_sms - 1) / (4 * num_sms);
    int rpc = (want + rows_step - 1) / rows_step * rows_step;
    if (rpc < rows_step) rpc = rows_step;
    cfg.gridDim = dim3((max_n + rpc - 1) / rpc, d.B, 1);
    cfg.blockDim = dim3(kScoreThreads, 1, 1);
    cfg.dynamicSmemBytes = (size_t)d.Q * d.E * sizeof(float);
    if (d.emb_dtype == LSA_BF16) {
        return cudaLaunchKernelEx(&cfg, k_score_stream<true>, (const uint8_t*)q_emb,
                                  (const uint8_t*)chunk_emb, scores, tab, d.Q, d.E, rpc);
    }
    return cudaLaunchKernelEx(&cfg, k_score_stream<false>, (const uint8_t*)q_emb,
                              (const uint8_t*)chunk_emb, scores, tab, d.Q, d.E, rpc);
}

}  // namespace lsa
