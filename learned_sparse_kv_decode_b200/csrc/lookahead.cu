// lookahead.cu - attention of every lookahead-window query over the kept chunks, on the
// tensor cores (tcgen05).
//
// FlashMemory-DeepSeek-V4 (review on dimensionstp.github.io, section 3-2 (3)): the indexer
// keeps the chunks that the next ~64 tokens will attend to, and until the next retrieval
// cycle those tokens attend over the kept chunks only (steps 6-7). With the whole window's
// queries at hand, for sequence b, head h and window query j:
//     out[b][j][h] = sum_t softmax_t(q[b][j][h] . K_t[h] / sqrt(Dh)) V_t[h]   over kept tokens t
//     lse[b][j][h] = log sum_t exp(q[b][j][h] . K_t[h] / sqrt(Dh))
//
// The Qw <= 64 queries of a (sequence, head) share every K/V row: 2*2*Qw flops per K/V
// element, 64 flop per byte at Qw = 64. That is still HBM-bound on the tensor pipe, but far
// beyond what the CUDA cores sustain at HBM speed, so both products run as tcgen05 MMAs.
//
// One CTA per SM, persistent over a balanced run of tiles:
//  * A tile is 64 consecutive kept tokens of one (sequence, head). The tiles of all (b, h)
//    form one global list; CTA c takes tiles [c*S/G, (c+1)*S/G) (split-K over the list).
//  * Warp 4 (producer) streams each tile's K and V rows from the full cache, through the
//    kept chunk ids (or from a compact resident buffer), with 3-D TMA tile loads into a
//    5-deep ring in the 128-byte-swizzled layout the MMAs read. No multicast; L2 evict-first.
//  * Warp 5 (one thread) issues the MMAs:
//      S  = Qd . K^T   M = 128, N = 64,  K = 128  bf16 -> fp32 TMEM, double-buffered
//      O += P . V      M = 128, N = 128, K = 64   P from shared memory, V MN-major
//    Qd holds the window's queries twice (rows 0-63 and 64-127). Rows 0-63 use the scores
//    of the tile's tokens 0-31 and rows 64-127 those of tokens 32-63 (their P is zero over
//    the other half). So each of the 128 softmax threads owns one (query, half-tile) row,
//    and all four TMEM lane quarters do work. The MMAs do twice the useful flops; at 128
//    flop per K/V byte that still sits well under the tensor-pipe roofline.
//  * Warps 0-3 (softmax) handle one row per thread. Each thread reads its 32 scores
//    (tcgen05.ld) and keeps a running max m and sum l in the log2 domain. It writes its bf16
//    P row to shared memory; l sums the rounded P actually used. It rescales its O row in
//    TMEM only when m grows by more than 8 (2^8); a stale max is exact after the final
//    division by l.
//  * At the end of a (b, h) run the two half-rows of each query merge in the CTA
//    (log-sum-exp). A run wholly inside the CTA writes out/lse directly. A run split across
//    CTAs writes a partial (O, m, l) to slot 2c (the CTA's first run) or 2c + 1 (its last
//    run); k_attn_la_merge combines them.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>

#include "lsa_device.cuh"

namespace lsa {

namespace la {
constexpr int kTile = 64;                 // kept tokens per tile
constexpr int kRows = 128;                // MMA rows: the window's queries, twice
constexpr int kQmax = 64;                 // window queries per (sequence, head)
constexpr int kStages = 5;                // K/V ring depth
constexpr uint32_t kHalf = kTile * 128;   // a 64-dim half of a K or V tile: 64 rows x 128 B
constexpr uint32_t kOperand = 2 * kHalf;  // a K or V tile (16 KiB)
constexpr uint32_t kStage = 2 * kOperand; // K + V (32 KiB)
constexpr uint32_t kQHalf = kRows * 128;  // a 64-dim half of Qd (16 KiB)
constexpr uint32_t kQBytes = 2 * kQHalf;  // Qd (32 KiB)
constexpr uint32_t kPBytes = kRows * 128; // a P tile: 128 rows x 64 tokens bf16 (16 KiB)
constexpr uint32_t kSmem = kQBytes + 2 * kPBytes + kStages * kStage + 1024;  // + alignment slack
constexpr int kThreads = 192;             // warps 0-3 softmax, 4 producer, 5 MMA
constexpr uint32_t kTmemCols = 256;       // S: 2 x 64 columns, then O: 128 columns
constexpr uint32_t kTmemO = 128;          // first O column
constexpr float kRescale = 8.0f;          // lazy-rescale threshold (log2 units)
constexpr float kLn2 = 0.69314718055994531f;
static_assert(kQBytes % 1024 == 0 && kPBytes % 1024 == 0 && kStage % 1024 == 0, "1 KiB swizzle atoms");
}  // namespace la

struct LaParams {
    int32_t H;        // heads
    int32_t Qw;       // window queries (1..64)
    int32_t G;        // CTAs
    int32_t indexed;  // K/V read through chunk ids (1) or from compact resident buffers (0)
    int32_t boxh;     // token rows per TMA box: min(C, 64)
    int32_t nbox;     // boxes per tile: 64 / boxh
    int64_t S;        // tiles in the global list
    float qscale;     // log2(e) / sqrt(Dh)
    int32_t tile_off[kMaxB + 1];  // first tile of each sequence (its H runs follow in head order)
};

// Position in the tile list: run (b, h), tile t of the run.
struct LaCursor {
    int b, h, t;
    int nt;  // tiles per run of sequence b
    int kt;  // kept tokens of sequence b
};

__device__ __forceinline__ void la_seq(LaCursor& u, int b, const SeqTable& tab) {
    u.b = b;
    u.kt = (tab.kept_off[b + 1] - tab.kept_off[b]) * tab.C;
    u.nt = (u.kt + la::kTile - 1) / la::kTile;
}

__device__ __forceinline__ LaCursor la_cursor(int64_t s, const SeqTable& tab, const LaParams& lp) {
    LaCursor u;
    la_seq(u, seq_of(lp.tile_off, tab.B, s), tab);
    const int r = (int)(s - lp.tile_off[u.b]);
    u.h = r / u.nt;
    u.t = r - u.h * u.nt;
    return u;
}

__device__ __forceinline__ void la_next(LaCursor& u, const SeqTable& tab, const LaParams& lp) {
    if (++u.t < u.nt) return;
    u.t = 0;
    if (++u.h < lp.H) return;
    u.h = 0;
    if (u.b + 1 < tab.B) la_seq(u, u.b + 1, tab);
}

__host__ __device__ __forceinline__ int64_t la_cta_of_tile(int64_t s, int64_t S, int G) {
    return ((s + 1) * G + S - 1) / S - 1;
}

// Token row (in the K/V tensor) of box j of global tile s. A box past the sequence's kept
// tokens (a ragged last tile, C < 64) reloads a kept chunk; the softmax masks its scores.
__device__ __forceinline__ int la_box_row(int64_t s, int j, const int32_t* __restrict__ ids,
                                          const SeqTable& tab, const LaParams& lp, uint32_t* err) {
    const LaCursor u = la_cursor(s, tab, lp);
    const int kb = tab.kept_off[u.b + 1] - tab.kept_off[u.b];
    const int u0 = u.t * la::kTile + j * lp.boxh;  // kept-token position within the sequence
    int kc = u0 / tab.C, off = u0 - kc * tab.C;
    if (kc >= kb) {
        kc = kb - 1;
        off = 0;
    }
    if (!lp.indexed) return (tab.kept_off[u.b] + kc) * tab.C + off;
    int32_t id = ids[tab.kept_off[u.b] + kc];
    const int nb = tab.chunk_off[u.b + 1] - tab.chunk_off[u.b];
    if (id < 0 || id >= nb) {
        set_error(err, kErrBadId);
        id = 0;
    }
    return (tab.chunk_off[u.b] + id) * tab.C + off;
}

// ------------------------------------------------------------------ tcgen05 / TMA helpers
// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 layout type 2): 128-byte rows,
// 8-row atoms of 1 KiB (SBO = 1024). A K-major operand ignores LBO (encoded 1); for an
// MN-major operand LBO is the distance between its 64-element column blocks.
__device__ __forceinline__ uint64_t la_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// kind::f16 instruction descriptor: bf16 A (K-major) and B (K-major or MN-major), fp32 D.
__host__ __device__ constexpr uint32_t la_idesc(int M, int N, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (b_mn ? (1u << 16) : 0u) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void la_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

__device__ __forceinline__ void la_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void la_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void la_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void la_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void la_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
        "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void la_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void la_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 3-D TMA tile load (no multicast) with an L2 cache hint.
__device__ __forceinline__ void la_tma3(uint32_t dst, const CUtensorMap* map, int x, int y, int z, uint32_t bar,
                                        uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar), "l"(pol)
        : "memory");
}

// 4-D TMA tile load (no multicast).
__device__ __forceinline__ void la_tma4(uint32_t dst, const CUtensorMap* map, int x, int y, int z, int w,
                                        uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void la_sts128(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ float la_ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void la_softmax_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Bounded wait by a whole warp; the result is warp-uniform. Once a wait gives up (or another
// role gave up), the CTA's roles skip their remaining waits and work but keep their barriers.
__device__ __forceinline__ bool la_wait_warp(bool dead, uint32_t bar, uint32_t parity, uint32_t* err,
                                             int* abort_flag) {
    bool d = dead || *(volatile int*)abort_flag != 0;
    if (!d && !mbar_wait(bar, parity, err)) {
        d = true;
        *(volatile int*)abort_flag = 1;
    }
    return __any_sync(0xffffffffu, d);
}

// ------------------------------------------------------------------ the kernel
// grid (G), la::kThreads threads, dynamic smem la::kSmem.
// tmQ: q [B][Qw][H][Dh] bf16, box {64, 1, 64, 1}; tmK / tmV: [rows][H][Dh] bf16, box {64, 1, boxh};
// all 128-byte swizzled.
__global__ void __launch_bounds__(la::kThreads, 1)
k_attn_la(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
          const __grid_constant__ CUtensorMap tmV, const int32_t* __restrict__ ids, float* __restrict__ out,
          float* __restrict__ lse, float* __restrict__ part_o, float* __restrict__ part_ml, const SeqTable tab,
          const LaParams lp, uint32_t* err) {
    using namespace la;
    extern __shared__ uint8_t la_raw[];
    __shared__ __align__(8) uint64_t bar_kf[kStages], bar_vf[kStages], bar_ke[kStages];
    __shared__ __align__(8) uint64_t bar_sf[2], bar_pf[2], bar_od[2];
    __shared__ __align__(8) uint64_t bar_qf, bar_qe, bar_end;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    __shared__ float2 s_ml[kQmax];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = blockIdx.x;
    const int64_t s0 = (int64_t)c * lp.S / lp.G, s1 = (int64_t)(c + 1) * lp.S / lp.G;
    const int64_t n = s1 - s0;
    const uint32_t raw = smem_u32(la_raw);
    const uint32_t sQ = (raw + 1023u) & ~1023u;
    const uint32_t sP = sQ + kQBytes, sKV = sP + 2 * kPBytes;
    const uint32_t kf0 = smem_u32(bar_kf), vf0 = smem_u32(bar_vf), ke0 = smem_u32(bar_ke);
    const uint32_t sf0 = smem_u32(bar_sf), pf0 = smem_u32(bar_pf), od0 = smem_u32(bar_od);
    const uint32_t qf = smem_u32(&bar_qf), qe = smem_u32(&bar_qe), endb = smem_u32(&bar_end);

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(kf0 + 8 * i, 1);
            mbar_init(vf0 + 8 * i, 1);
            mbar_init(ke0 + 8 * i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(sf0 + 8 * i, 1);
            mbar_init(pf0 + 8 * i, 128);
            mbar_init(od0 + 8 * i, 1);
        }
        mbar_init(qf, 1);
        mbar_init(qe, 1);
        mbar_init(endb, 1);
        fence_mbar_init();
        s_abort = 0;
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    la_fence_before();
    __syncthreads();
    la_fence_after();
    const uint32_t tmem = s_tmem;
    pdl_trigger();

    if (warp == 4) {
        // ------------------------------------------------ producer (lane 0 issues, the warp resolves rows)
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmQ)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmK)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmV)) : "memory");
        }
        const uint64_t pol = policy_evict_first();
        pdl_wait();  // chunk ids come from the preceding kernel
        const int64_t npairs = n * lp.nbox;  // (tile, box) pairs of this CTA
        LaCursor cur = la_cursor(s0, tab, lp);
        bool dead = false;
        int64_t issued = 0;  // tiles whose loads were all issued
        int qloads = 0;
        for (int64_t p0 = 0; p0 < npairs && !dead; p0 += 32) {
            int row = 0;
            if (p0 + lane < npairs) {
                const int64_t p = p0 + lane;
                row = la_box_row(s0 + p / lp.nbox, (int)(p % lp.nbox), ids, tab, lp, err);
            }
            const int cnt = (int)(npairs - p0 < 32 ? npairs - p0 : 32);
            for (int qq = 0; qq < cnt; ++qq) {
                const int rq = __shfl_sync(0xffffffffu, row, qq);
                if (lane == 0 && !dead) {
                    const int64_t i = (p0 + qq) / lp.nbox;
                    const int j = (int)((p0 + qq) % lp.nbox);
                    const int st = (int)(i % kStages);
                    if (j == 0) {
                        if (*(volatile int*)&s_abort) dead = true;
                        if (!dead && (i == 0 || cur.t == 0)) {
                            // a run starts: its queries replace the previous run's once those S are done
                            if (qloads > 0 && !mbar_wait(qe, (uint32_t)(qloads - 1) & 1u, err)) dead = true;
                            if (!dead) {
                                mbar_arrive_expect_tx(qf, kQBytes);
                                for (int d = 0; d < 2; ++d)
                                    for (int rr = 0; rr < 2; ++rr)
                                        la_tma4(sQ + d * kQHalf + rr * (kQHalf / 2), &tmQ, 64 * d, cur.h, 0, cur.b, qf);
                                ++qloads;
                            }
                        }
                        if (!dead && !mbar_wait(ke0 + 8 * st, ((uint32_t)(i / kStages) & 1u) ^ 1u, err)) dead = true;
                        if (!dead) {
                            mbar_arrive_expect_tx(kf0 + 8 * st, kOperand);
                            mbar_arrive_expect_tx(vf0 + 8 * st, kOperand);
                        }
                    }
                    if (!dead) {
                        const uint32_t kd = sKV + (uint32_t)st * kStage + (uint32_t)j * lp.boxh * 128;
                        const uint32_t vd = kd + kOperand;
                        la_tma3(kd, &tmK, 0, cur.h, rq, kf0 + 8 * st, pol);
                        la_tma3(kd + kHalf, &tmK, 64, cur.h, rq, kf0 + 8 * st, pol);
                        la_tma3(vd, &tmV, 0, cur.h, rq, vf0 + 8 * st, pol);
                        la_tma3(vd + kHalf, &tmV, 64, cur.h, rq, vf0 + 8 * st, pol);
                        if (j == lp.nbox - 1) {
                            ++issued;
                            la_next(cur, tab, lp);
                        }
                    } else {
                        s_abort = 1;
                    }
                }
                dead = __shfl_sync(0xffffffffu, dead ? 1 : 0, 0) != 0;
                if (dead) break;
            }
        }
        if (lane == 0) {
            // the copies still in flight land before the CTA may exit
            for (int64_t i = issued > kStages ? issued - kStages : 0; i < issued; ++i) {
                const uint32_t par = (uint32_t)(i / kStages) & 1u;
                mbar_wait(kf0 + 8 * (uint32_t)(i % kStages), par, err);
                mbar_wait(vf0 + 8 * (uint32_t)(i % kStages), par, err);
            }
            if (qloads > 0) mbar_wait(qf, (uint32_t)(qloads - 1) & 1u, err);
        }
    } else if (warp == 5) {
        // ------------------------------------------------ MMA issuer (one thread)
        if (lane == 0) {
            const uint32_t idS = la_idesc(kRows, kTile, false), idO = la_idesc(kRows, kDh, true);
            LaCursor cs = la_cursor(s0, tab, lp), co = cs;
            int qwaits = 0;
            bool dead = false;
            // S of tile i into TMEM columns (i & 1) * 64
            auto issue_s = [&](int64_t i, const LaCursor& u) -> bool {
                if (i == 0 || u.t == 0) {  // a run starts: its queries must have landed
                    if (!mbar_wait(qf, (uint32_t)qwaits & 1u, err)) return false;
                    ++qwaits;
                }
                const int st = (int)(i % kStages);
                if (!mbar_wait(kf0 + 8 * st, (uint32_t)(i / kStages) & 1u, err)) return false;
                la_fence_after();
                const uint32_t kb = sKV + (uint32_t)st * kStage;
#pragma unroll
                for (int kk = 0; kk < kDh / 16; ++kk) {
                    const uint64_t a = la_desc(sQ + (uint32_t)(kk >> 2) * kQHalf + (uint32_t)(kk & 3) * 32, 16, 1024);
                    const uint64_t b = la_desc(kb + (uint32_t)(kk >> 2) * kHalf + (uint32_t)(kk & 3) * 32, 16, 1024);
                    la_mma(tmem + (uint32_t)(i & 1) * kTile, a, b, idS, kk > 0 ? 1u : 0u);
                }
                la_commit(sf0 + 8 * (uint32_t)(i & 1));
                if (i == n - 1 || u.t == u.nt - 1) la_commit(qe);  // the run's last S: Qd may be replaced
                return true;
            };
            if (n > 0 && !issue_s(0, cs)) dead = true;
            for (int64_t i = 0; i < n && !dead; ++i) {
                if (*(volatile int*)&s_abort) {
                    dead = true;
                    break;
                }
                if (i + 1 < n) {
                    la_next(cs, tab, lp);
                    if (!issue_s(i + 1, cs)) {
                        dead = true;
                        break;
                    }
                }
                const int st = (int)(i % kStages);
                if (!mbar_wait(pf0 + 8 * (uint32_t)(i & 1), (uint32_t)(i >> 1) & 1u, err) ||
                    !mbar_wait(vf0 + 8 * st, (uint32_t)(i / kStages) & 1u, err)) {
                    dead = true;
                    break;
                }
                la_fence_after();
                const bool first = (i == 0) || co.t == 0;
                const uint32_t pa = sP + (uint32_t)(i & 1) * kPBytes;
                const uint32_t vb = sKV + (uint32_t)st * kStage + kOperand;
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk) {
                    const uint64_t a = la_desc(pa + (uint32_t)kk * 32, 16, 1024);
                    const uint64_t b = la_desc(vb + (uint32_t)kk * 2048, kHalf, 1024);
                    la_mma(tmem + kTmemO, a, b, idO, (!first || kk > 0) ? 1u : 0u);
                }
                la_commit(od0 + 8 * (uint32_t)(i & 1));
                la_commit(ke0 + 8 * st);
                la_next(co, tab, lp);
            }
            if (dead) s_abort = 1;
            // every MMA issued has completed before TMEM is released
            la_commit(endb);
            mbar_wait(endb, 0, err);
        }
    } else {
        // ------------------------------------------------ softmax: thread r owns TMEM lane r
        const int r = tid, half = r >> 6, qrow = r & 63;
        const uint32_t lane_t = tmem + ((uint32_t)(warp * 32) << 16);
        const uint32_t prow = (uint32_t)(r >> 3) * 1024 + (uint32_t)(r & 7) * 128;
        float* scratch = reinterpret_cast<float*>(la_raw + (sP - raw));  // both P tiles, at run ends
        LaCursor cur = la_cursor(s0, tab, lp);
        float m = -INFINITY, l = 0.f;
        bool dead = false, run_whole = false;
        int run_idx = 0;
        for (int64_t i = 0; i < n; ++i) {
            const bool first = (i == 0) || cur.t == 0;
            const bool last = (i == n - 1) || cur.t == cur.nt - 1;
            if (first) {
                m = -INFINITY;
                l = 0.f;
                run_whole = cur.t == 0;
            }
            // 1. this row's 32 scores of tile i
            dead = la_wait_warp(dead, sf0 + 8 * (uint32_t)(i & 1), (uint32_t)(i >> 1) & 1u, err, &s_abort);
            la_fence_after();
            uint32_t sr[32];
            if (!dead) {
                la_ld32(lane_t + (uint32_t)(i & 1) * kTile + (uint32_t)half * 32, sr);
                la_wait_ld();
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) sr[j] = 0u;
            }
            const int rem = cur.kt - (cur.t * kTile + half * 32);
            const int nvalid = rem < 0 ? 0 : (rem > 32 ? 32 : rem);
            float x[32], mt = -INFINITY;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                x[j] = j < nvalid ? __uint_as_float(sr[j]) * lp.qscale : -INFINITY;
                mt = fmaxf(mt, x[j]);
            }
            // 2. running max; O is rescaled only when the max grows past the threshold
            const float mn = fmaxf(m, mt);
            float alpha = 1.f;
            bool need = false;
            if (first) {
                m = mn;
            } else if (mn > m + kRescale) {
                need = true;
                alpha = la_ex2(m - mn);
                m = mn;
            }
            if (__any_sync(0xffffffffu, need)) {
                dead = la_wait_warp(dead, od0 + 8 * (uint32_t)((i - 1) & 1), (uint32_t)((i - 1) >> 1) & 1u, err,
                                    &s_abort);
                la_fence_after();
                if (!dead) {
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        uint32_t o[32];
                        la_ld32(lane_t + kTmemO + (uint32_t)cc * 32, o);
                        la_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
                        la_st32(lane_t + kTmemO + (uint32_t)cc * 32, o);
                    }
                    la_wait_st();
                }
                l *= alpha;
            }
            // 3. P of tile i into P tile (i & 1), free once O(i - 2) has completed
            if (i >= 2)
                dead = la_wait_warp(dead, od0 + 8 * (uint32_t)(i & 1), (uint32_t)((i - 2) >> 1) & 1u, err, &s_abort);
            uint32_t pk[16];
            float ps = 0.f;
            const bool live = m != -INFINITY;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float p0 = live ? la_ex2(x[2 * j] - m) : 0.f;
                const float p1 = live ? la_ex2(x[2 * j + 1] - m) : 0.f;
                const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                pk[j] = *reinterpret_cast<const uint32_t*>(&h2);
                ps += bf16lo(pk[j]) + bf16hi(pk[j]);
            }
            l += ps;
            const uint32_t pb = sP + (uint32_t)(i & 1) * kPBytes + prow;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if ((cc >> 2) == half) {
                    const int b4 = (cc & 3) * 4;
                    v = make_uint4(pk[b4], pk[b4 + 1], pk[b4 + 2], pk[b4 + 3]);
                }
                la_sts128(pb + ((uint32_t)(cc ^ (r & 7)) << 4), v);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            la_fence_before();
            mbar_arrive(pf0 + 8 * (uint32_t)(i & 1));

            // 4. end of this CTA's part of run (b, h): merge the half-rows, write out or a partial
            if (last) {
                dead = la_wait_warp(dead, od0 + 8 * (uint32_t)(i & 1), (uint32_t)(i >> 1) & 1u, err, &s_abort);
                la_fence_after();
                const bool whole = run_whole && cur.t == cur.nt - 1;
                if (half == 1) {
                    s_ml[qrow] = make_float2(m, l);
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        uint32_t o[32];
                        if (!dead) {
                            la_ld32(lane_t + kTmemO + (uint32_t)cc * 32, o);
                            la_wait_ld();
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j) o[j] = 0u;
                        }
#pragma unroll
                        for (int j = 0; j < 32; ++j) scratch[(cc * 32 + j) * kQmax + qrow] = __uint_as_float(o[j]);
                    }
                }
                la_softmax_sync();
                if (half == 0) {
                    const float2 o2 = s_ml[qrow];
                    const float M = fmaxf(m, o2.x);
                    const float wa = m == -INFINITY ? 0.f : la_ex2(m - M);
                    const float wb = o2.x == -INFINITY ? 0.f : la_ex2(o2.x - M);
                    const float L = wa * l + wb * o2.y;
                    const bool wr = qrow < lp.Qw && !dead;
                    const int64_t slot = 2 * (int64_t)c + (run_idx == 0 ? 0 : 1);
                    float* dst = whole ? out + (((int64_t)cur.b * lp.Qw + qrow) * lp.H + cur.h) * kDh
                                       : part_o + (slot * lp.Qw + qrow) * kDh;
                    const float inv = whole ? 1.f / L : 1.f;
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        uint32_t o[32];
                        if (!dead) {
                            la_ld32(lane_t + kTmemO + (uint32_t)cc * 32, o);
                            la_wait_ld();
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j) o[j] = 0u;
                        }
                        if (wr) {
#pragma unroll
                            for (int j = 0; j < 32; j += 4) {
                                float4 v;
                                v.x = (wa * __uint_as_float(o[j]) + wb * scratch[(cc * 32 + j) * kQmax + qrow]) * inv;
                                v.y = (wa * __uint_as_float(o[j + 1]) + wb * scratch[(cc * 32 + j + 1) * kQmax + qrow]) * inv;
                                v.z = (wa * __uint_as_float(o[j + 2]) + wb * scratch[(cc * 32 + j + 2) * kQmax + qrow]) * inv;
                                v.w = (wa * __uint_as_float(o[j + 3]) + wb * scratch[(cc * 32 + j + 3) * kQmax + qrow]) * inv;
                                *reinterpret_cast<float4*>(dst + cc * 32 + j) = v;
                            }
                        }
                    }
                    if (wr) {
                        if (whole) {
                            if (lse != nullptr)
                                lse[((int64_t)cur.b * lp.Qw + qrow) * lp.H + cur.h] = (M + log2f(L)) * kLn2;
                        } else {
                            *reinterpret_cast<float2*>(part_ml + (slot * lp.Qw + qrow) * 2) = make_float2(M, L);
                        }
                    }
                }
                la_softmax_sync();  // the scratch is read before the next P tile is written
                ++run_idx;
            }
            la_next(cur, tab, lp);
        }
    }

    la_fence_before();
    __syncthreads();
    if (warp == 0) {
        la_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(la::kTmemCols)
                     : "memory");
    }
}

// Merge of the partials of the runs split across CTAs (log-sum-exp rule). grid (B*H, ceil(Qw/8)),
// 256 threads: warp w merges window query blockIdx.y*8 + w; lane k owns output columns 4k..4k+3.
__global__ void __launch_bounds__(256)
k_attn_la_merge(const float* __restrict__ part_o, const float* __restrict__ part_ml, float* __restrict__ out,
                float* __restrict__ lse, const SeqTable tab, const LaParams lp) {
    const int g = blockIdx.x, b = g / lp.H, h = g - b * lp.H;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = blockIdx.y * 8 + w;
    pdl_wait();
    if (q >= lp.Qw) return;
    const int kt = (tab.kept_off[b + 1] - tab.kept_off[b]) * tab.C;
    const int nt = (kt + la::kTile - 1) / la::kTile;
    const int64_t ts = lp.tile_off[b] + (int64_t)h * nt, te = ts + nt;
    const int c0 = (int)la_cta_of_tile(ts, lp.S, lp.G), c1 = (int)la_cta_of_tile(te - 1, lp.S, lp.G);
    if (c0 == c1) return;  // written directly by its CTA
    const int ns = c1 - c0 + 1;
    // the run is the first run of every CTA after c0; of c0 only if c0's tiles start inside it
    const int slot0 = 2 * c0 + (((int64_t)c0 * lp.S / lp.G) >= ts ? 0 : 1);
    auto slot_of = [&](int i) { return i == 0 ? slot0 : 2 * (c0 + i); };

    float M = -INFINITY;
    for (int i = lane; i < ns; i += 32) M = fmaxf(M, part_ml[((int64_t)slot_of(i) * lp.Qw + q) * 2]);
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i0 = 0; i0 < ns; i0 += 32) {
        float wgt = 0.f;
        if (i0 + lane < ns) {
            const float2 ml = *reinterpret_cast<const float2*>(part_ml + ((int64_t)slot_of(i0 + lane) * lp.Qw + q) * 2);
            wgt = ml.x == -INFINITY ? 0.f : la_ex2(ml.x - M);
            L = fmaf(wgt, ml.y, L);
        }
        const int cnt = ns - i0 < 32 ? ns - i0 : 32;
        for (int jj = 0; jj < cnt; ++jj) {
            const float wj = __shfl_sync(0xffffffffu, wgt, jj);
            const float4 v = *reinterpret_cast<const float4*>(part_o + ((int64_t)slot_of(i0 + jj) * lp.Qw + q) * kDh +
                                                              lane * 4);
            acc.x = fmaf(wj, v.x, acc.x);
            acc.y = fmaf(wj, v.y, acc.y);
            acc.z = fmaf(wj, v.z, acc.z);
            acc.w = fmaf(wj, v.w, acc.w);
        }
    }
    for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
    const float inv = 1.f / L;
    float* dst = out + (((int64_t)b * lp.Qw + q) * lp.H + h) * kDh + lane * 4;
    *reinterpret_cast<float4*>(dst) = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    if (lse != nullptr && lane == 0) lse[((int64_t)b * lp.Qw + q) * lp.H + h] = (M + log2f(L)) * la::kLn2;
}

// ------------------------------------------------------------------ host side
namespace {

PFN_cuTensorMapEncodeTiled_v12000 la_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (encode == nullptr) {
        cudaDriverEntryPointQueryResult q;
        void* fn = nullptr;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || fn == nullptr) return nullptr;
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    return encode;
}

// A bf16 tensor whose innermost dimension is the head dimension (256-byte rows), read in
// boxes of 64 elements (128 bytes) x the given outer extents, 128-byte swizzle, zero fill.
cudaError_t la_tmap(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims, const cuuint32_t* box) {
    PFN_cuTensorMapEncodeTiled_v12000 encode = la_encoder();
    if (encode == nullptr) return cudaErrorInvalidValue;
    cuuint64_t strides[3];
    cuuint64_t s = (cuuint64_t)dims[0] * 2;
    for (int i = 1; i < rank; ++i) {
        strides[i - 1] = s;
        s *= dims[i];
    }
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

int la_smem_bytes() { return (int)la::kSmem; }
int la_max_queries() { return la::kQmax; }

cudaError_t la_init_attrs(int* ctas_per_sm) {
    cudaError_t e = set_smem_attrs(k_attn_la, (int)la::kSmem);
    if (e == cudaSuccess) e = set_smem_attrs(k_attn_la_merge, 0);
    if (e != cudaSuccess) return e;
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_attn_la, la::kThreads, la::kSmem);
    if (e != cudaSuccess) return e;
    *ctas_per_sm = occ;
    return cudaSuccess;
}

// Tiles of the global list (sum over sequences of H * ceil(k_b * C / 64)).
int64_t la_tiles(const lsa_dims& d, const SeqTable& tab) {
    int64_t S = 0;
    for (int b = 0; b < d.B; ++b) {
        const int64_t kt = (int64_t)(tab.kept_off[b + 1] - tab.kept_off[b]) * tab.C;
        S += (int64_t)d.H * ((kt + la::kTile - 1) / la::kTile);
    }
    return S;
}

// q [B][Qw][H][Dh], K/V [kv_rows][H][Dh] bf16; ids (or nullptr: compact resident buffers);
// part_o [2*max_ctas][Qw][Dh] and part_ml [2*max_ctas][Qw][2] fp32 workspace.
cudaError_t launch_attention_la(const lsa_dims& d, const SeqTable& tab, int max_ctas, const void* q, const void* K,
                                const void* V, int64_t kv_rows, const int32_t* ids, float* part_o, float* part_ml,
                                float* out, float* lse, uint32_t* err, cudaStream_t stream, bool pdl) {
    LaParams lp;
    std::memset(&lp, 0, sizeof(lp));
    lp.H = d.H;
    lp.Qw = d.Q;
    lp.boxh = d.chunk_len < la::kTile ? d.chunk_len : la::kTile;
    lp.nbox = la::kTile / lp.boxh;
    int64_t S = 0;
    for (int b = 0; b < d.B; ++b) {
        lp.tile_off[b] = (int32_t)S;
        const int64_t kt = (int64_t)(tab.kept_off[b + 1] - tab.kept_off[b]) * tab.C;
        S += (int64_t)d.H * ((kt + la::kTile - 1) / la::kTile);
    }
    lp.tile_off[d.B] = (int32_t)S;
    lp.S = S;
    lp.G = (int)(S < max_ctas ? S : max_ctas);
    lp.indexed = ids != nullptr ? 1 : 0;
    lp.qscale = 1.4426950408889634f / sqrtf((float)kDh);

    alignas(64) CUtensorMap tq, tk, tv;
    {
        const cuuint64_t dq[4] = {(cuuint64_t)kDh, (cuuint64_t)d.H, (cuuint64_t)d.Q, (cuuint64_t)d.B};
        const cuuint32_t bq[4] = {64, 1, (cuuint32_t)la::kQmax, 1};
        cudaError_t e = la_tmap(&tq, q, 4, dq, bq);
        if (e != cudaSuccess) return e;
        const cuuint64_t dkv[3] = {(cuuint64_t)kDh, (cuuint64_t)d.H, (cuuint64_t)kv_rows};
        const cuuint32_t bkv[3] = {64, 1, (cuuint32_t)lp.boxh};
        e = la_tmap(&tk, K, 3, dkv, bkv);
        if (e == cudaSuccess) e = la_tmap(&tv, V, 3, dkv, bkv);
        if (e != cudaSuccess) return e;
    }

    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    cfg.gridDim = dim3(lp.G, 1, 1);
    cfg.blockDim = dim3(la::kThreads, 1, 1);
    cfg.dynamicSmemBytes = la::kSmem;
    cudaError_t e = cudaLaunchKernelEx(&cfg, k_attn_la, tq, tk, tv, ids, out, lse, part_o, part_ml, tab, lp, err);
    if (e != cudaSuccess) return e;

    cudaLaunchConfig_t mc = {};
    mc.stream = stream;
    mc.attrs = attr;
    mc.numAttrs = 1;
    mc.gridDim = dim3(d.B * d.H, (d.Q + 7) / 8, 1);
    mc.blockDim = dim3(256, 1, 1);
    mc.dynamicSmemBytes = 0;
    const float* cpo = part_o;
    const float* cpm = part_ml;
    return cudaLaunchKernelEx(&mc, k_attn_la_merge, cpo, cpm, out, lse, tab, lp);
}

}  // namespace lsa
