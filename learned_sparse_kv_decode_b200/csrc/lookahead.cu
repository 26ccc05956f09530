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
// One CTA per SM, persistent over one contiguous range of tiles:
//  * A tile is 128 consecutive kept tokens of one (sequence, head). The tiles of all (b, h)
//    form one global list split over the CTAs by cost (split-K over the list): a tile costs 1
//    and the start of a (b, h) run 4 more, since a CTA that switches runs reloads its queries
//    and merges the finished run. The host computes the ranges (la_partition) and passes them
//    in the kernel parameters.
//  * Warp 8 (producer) streams each tile's K and V rows from the full cache, through the
//    kept chunk ids (or from a compact resident buffer), with 3-D TMA tile loads in the
//    128-byte-swizzled layout the MMAs read: a 2-deep K ring (a K tile is free once its S has
//    completed) and a 4-deep V ring (free only once its O has, after the tile's softmax: the
//    longer-held operand gets the deeper ring). No multicast; L2 evict-first.
//  * Warp 9 (one thread) issues the MMAs as their inputs arrive (polling, never blocking on
//    one barrier while another product is ready):
//      S  = Q . K^T    M = 64, N = 128, K = 128  bf16 -> fp32 TMEM, 2 buffers
//      O += P . V      M = 64, N = 128, K = 128  P read from TMEM, V an MN-major smem operand
//    M = 64 holds the window's queries once. A tcgen05 MMA with N <= 128 takes about the same
//    time whatever its M (64 or 128) and N, so the tile is as wide as the S product allows;
//    M = 64 does half the multiply-adds of a 128-row product, and its 16 KiB of queries leave
//    room for a sixth ring stage.
//  * Warps 0-3 and 4-7 are two softmax groups that take alternate tiles. Each group has
//    its own running max m and sum l per row (log2 domain) and its own O accumulator in
//    TMEM, so two tiles' softmax overlap. An M = 64 accumulator keeps row m in TMEM lane
//    (m % 16) + 32 (m / 16); the 16-lane access shapes give each thread two rows and a quarter
//    of their columns, so the four threads of a quad share two rows (max by shuffles, each
//    thread sums the weights of its own tokens). A thread reads its scores (tcgen05.ld) and
//    writes its bf16 weights over the first 64 columns of the same S buffer (tcgen05.st); l
//    sums the fp32 weights. A row's O is rescaled only when its m grows by more than 8 (2^8);
//    a stale max is exact after the final division by l.
//  * Per S buffer, three mbarriers order the hand-offs: S landed, P written, and the O
//    product that read P completed. Each completes one phase every two tiles, and the
//    hand-offs keep every waiter within one phase of it (a parity wait two phases out of
//    step would pass early).
//  * At the end of a (b, h) run, group 0 merges its own and group 1's O rows straight from
//    TMEM (same lanes, log-sum-exp). A run wholly inside the CTA writes out/lse directly. A
//    run split across CTAs writes a partial (O, m, l) to slot 2c (the CTA's first run) or
//    2c + 1 (its last run), and k_attn_la_merge combines them.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>

#include "lsa_device.cuh"

namespace lsa {

namespace la {
constexpr int kTile = 128;                // kept tokens per tile
constexpr int kHalfTok = kTile / 2;       // tokens of a half tile (the bad-id mask is built 64 at a time)
constexpr int kRows = 64;                 // MMA rows (M = 64): the window's queries
constexpr int kQmax = 64;                 // window queries per (sequence, head)
constexpr int kKStages = 2;               // K ring depth (a K tile is free once its S has completed)
constexpr int kVStages = 4;               // V ring depth (a V tile is free once its O has completed)
constexpr uint32_t kHalf = kTile * 128;   // a 64-dim half of a K or V tile: 128 rows x 128 B (16 KiB)
constexpr uint32_t kOperand = 2 * kHalf;  // a K or V tile (32 KiB)

constexpr uint32_t kQHalf = kRows * 128;  // a 64-dim half of the queries (8 KiB)
constexpr uint32_t kQBytes = 2 * kQHalf;  // the queries (16 KiB)
constexpr uint32_t kSmem = kQBytes + (kKStages + kVStages) * kOperand + 1024;  // + alignment slack
constexpr int kThreads = 320;             // warps 0-7 softmax (two groups of 4), 8 producer, 9 MMA
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kSBufs = 2;                 // S buffers in TMEM (one per softmax group)
constexpr uint32_t kTmemCols = 512;       // S: 2 x 128 columns, then O of group 0 and of group 1
constexpr uint32_t kTmemO = kSBufs * kTile;  // first O column (group 0; group 1 follows)
constexpr float kRescale = 8.0f;          // lazy-rescale threshold (log2 units)
constexpr int kMaxCtas = 256;             // CTAs of one launch (one per SM)
constexpr int kRunCost = 4;               // extra cost of a run start in the tile split, in tiles (measured)
constexpr float kLn2 = 0.69314718055994531f;
static_assert(kQBytes % 1024 == 0 && kOperand % 1024 == 0, "1 KiB swizzle atoms");
static_assert(kTmemO + 2 * 128 == kTmemCols, "TMEM: S buffers then two O accumulators");

}  // namespace la

struct LaParams {
    int32_t H;        // heads
    int32_t Qw;       // window queries (1..64)
    int32_t G;        // CTAs
    int32_t indexed;  // K/V read through chunk ids (1) or from compact resident buffers (0)
    int32_t boxh;     // token rows per TMA box: min(C, 128)
    int32_t nbox;     // boxes per tile: 128 / boxh
    int64_t S;        // tiles in the global list
    float qscale;     // log2(e) / sqrt(Dh)
    int32_t tile_off[kMaxB + 1];        // first tile of each sequence (its H runs follow in head order)
    int32_t cta_start[la::kMaxCtas + 1];  // first tile of each CTA; cta_start[G] = S
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

// The CTA that owns tile s: the last c with cta_start[c] <= s (the ranges are non-empty).
__device__ __forceinline__ int la_cta_of(int64_t s, const LaParams& lp) {
    int lo = 0, hi = lp.G - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (lp.cta_start[mid] <= s) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Token row (in the K/V tensor) of box j of global tile s. A box past the sequence's kept
// tokens (a ragged last tile, C < 64) reloads a kept chunk, and a box of an out-of-range id
// loads chunk 0 of the sequence; the softmax masks the scores of both (la_bad_tokens).
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

// Tokens of the half tile that holds kept-token positions u0 .. u0 + 63 of run cursor u whose
// chunk id is out of range, as a 64-bit mask (bit j: position u0 + j). Positions past the kept
// tokens are left to the caller's count.
__device__ __forceinline__ uint64_t la_bad_tokens(const LaCursor& u, int u0, const int32_t* __restrict__ ids,
                                                  const SeqTable& tab) {
    const int kb = tab.kept_off[u.b + 1] - tab.kept_off[u.b];
    const int nb = tab.chunk_off[u.b + 1] - tab.chunk_off[u.b];
    uint64_t bad = 0;
    const int step = tab.C < la::kHalfTok ? tab.C : la::kHalfTok;  // tokens of one chunk inside the half
    for (int x = 0; x < la::kHalfTok; x += step) {
        const int kc = (u0 + x) / tab.C;
        if (kc >= kb) break;
        const int32_t id = ids[tab.kept_off[u.b] + kc];
        if (id < 0 || id >= nb) bad |= (step == 64 ? ~0ull : ((1ull << step) - 1ull)) << x;
    }
    return bad;
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

// D (TMEM) += A (TMEM, K-major: row = lane, two bf16 per 32-bit column) . B (shared memory).
__device__ __forceinline__ void la_mma_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
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

// The M = 64 accumulators (S, O) and the P operand hold row m in TMEM lane (m % 16) + 32 (m / 16):
// lanes 0-15 of each warp's 32-lane quarter. The 16-lane access shapes spread those 16 lanes over
// the warp's 32 threads; for thread t of the warp, per 8-column (.16x256b) or 4-column (.16x128b)
// block j of the access:
//   .16x256b: regs 4j, 4j+1 = lane t/4,     columns 8j + 2(t%4), 8j + 2(t%4) + 1
//             regs 4j+2, 4j+3 = lane t/4 + 8, the same columns
//   .16x128b: reg 2j = lane t/4, column 4j + t%4;  reg 2j+1 = lane t/4 + 8, the same column
// So a thread holds two rows (t/4 and t/4 + 8 of its quarter) and, of a 128-column row, the 32
// columns 8j + 2(t%4) + {0, 1}; the four threads of a quad (t/4 equal) share their two rows. Its two
// bf16 weights of block j (tokens 8j + 2(t%4) + {0, 1}) pack into P column 4j + t%4: exactly what
// .16x128b stores for it.

// 64 columns (8 blocks) of this thread's two rows, .16x256b.
__device__ __forceinline__ void la_ld256x8(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void la_st256x8(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.16x256b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

// 32 columns (8 blocks of 4) of this thread's two rows, .16x128b.
__device__ __forceinline__ void la_st128x8(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.16x128b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
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

__device__ __forceinline__ float la_ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Non-blocking probe of an mbarrier phase (mbarrier.try_wait may suspend the thread for a while,
// which would stall an issuer that polls several barriers).
__device__ __forceinline__ bool la_test_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ void la_softmax_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

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
    __shared__ __align__(8) uint64_t bar_kf[kKStages], bar_ke[kKStages];  // K ring full / empty
    __shared__ __align__(8) uint64_t bar_vf[kVStages], bar_ve[kVStages];  // V ring full / empty
    // per S buffer b: sf = S landed, pf = P written, sx = the O product reading that P has completed
    __shared__ __align__(8) uint64_t bar_sf[kSBufs], bar_pf[kSBufs], bar_sx[kSBufs];
    __shared__ __align__(8) uint64_t bar_qf, bar_qe, bar_end;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    __shared__ int s_anybad;          // some kept id of this CTA's tiles is out of range
    __shared__ float2 s_ml1[kRows];  // group 1's (m, l) per row, at a run end

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = blockIdx.x;
    const uint32_t raw = smem_u32(la_raw);
    const uint32_t sQ = (raw + 1023u) & ~1023u;
    const uint32_t sK = sQ + kQBytes, sV = sK + kKStages * kOperand;
    const uint32_t kf0 = smem_u32(bar_kf), ke0 = smem_u32(bar_ke), vf0 = smem_u32(bar_vf), ve0 = smem_u32(bar_ve);
    const uint32_t sf0 = smem_u32(bar_sf), pf0 = smem_u32(bar_pf), sx0 = smem_u32(bar_sx);
    const uint32_t qf = smem_u32(&bar_qf), qe = smem_u32(&bar_qe), endb = smem_u32(&bar_end);

    if (tid == 0) {
        for (int i = 0; i < kKStages; ++i) {
            mbar_init(kf0 + 8 * i, 1);
            mbar_init(ke0 + 8 * i, 1);
        }
        for (int i = 0; i < kVStages; ++i) {
            mbar_init(vf0 + 8 * i, 1);
            mbar_init(ve0 + 8 * i, 1);
        }
        for (int i = 0; i < kSBufs; ++i) {
            mbar_init(sf0 + 8 * i, 1);
            mbar_init(pf0 + 8 * i, 128);
            mbar_init(sx0 + 8 * i, 1);
        }
        mbar_init(qf, 1);
        mbar_init(qe, 1);
        mbar_init(endb, 1);
        fence_mbar_init();
        s_abort = 0;
        s_anybad = 0;
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
    const int64_t s0 = lp.cta_start[c], s1 = lp.cta_start[c + 1];
    const int n = (int)(s1 - s0);  // tiles of this CTA (the list is below 2^31 tiles)
    pdl_trigger();

    if (warp == kProducerWarp) {
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
                    const int sk = (int)(i % kKStages), sv = (int)(i % kVStages);
                    if (j == 0) {
                        if (*(volatile int*)&s_abort) dead = true;
                        if (!dead && (i == 0 || cur.t == 0)) {
                            // a run starts: its queries replace the previous run's once those S are done
                            if (qloads > 0 && !mbar_wait(qe, (uint32_t)(qloads - 1) & 1u, err)) dead = true;
                            if (!dead) {
                                mbar_arrive_expect_tx(qf, kQBytes);
                                for (int d = 0; d < 2; ++d) la_tma4(sQ + d * kQHalf, &tmQ, 64 * d, cur.h, 0, cur.b, qf);
                                ++qloads;
                            }
                        }
                        if (!dead && !mbar_wait(ke0 + 8 * sk, ((uint32_t)(i / kKStages) & 1u) ^ 1u, err)) dead = true;
                        if (!dead) mbar_arrive_expect_tx(kf0 + 8 * sk, kOperand);
                        if (!dead && !mbar_wait(ve0 + 8 * sv, ((uint32_t)(i / kVStages) & 1u) ^ 1u, err)) dead = true;
                        if (!dead) mbar_arrive_expect_tx(vf0 + 8 * sv, kOperand);
                    }
                    if (!dead) {
                        const uint32_t kd = sK + (uint32_t)sk * kOperand + (uint32_t)j * lp.boxh * 128;
                        const uint32_t vd = sV + (uint32_t)sv * kOperand + (uint32_t)j * lp.boxh * 128;
                        la_tma3(kd, &tmK, 0, cur.h, rq, kf0 + 8 * sk, pol);
                        la_tma3(kd + kHalf, &tmK, 64, cur.h, rq, kf0 + 8 * sk, pol);
                        la_tma3(vd, &tmV, 0, cur.h, rq, vf0 + 8 * sv, pol);
                        la_tma3(vd + kHalf, &tmV, 64, cur.h, rq, vf0 + 8 * sv, pol);
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
            for (int64_t i = issued > kKStages ? issued - kKStages : 0; i < issued; ++i)
                mbar_wait(kf0 + 8 * (uint32_t)(i % kKStages), (uint32_t)(i / kKStages) & 1u, err);
            for (int64_t i = issued > kVStages ? issued - kVStages : 0; i < issued; ++i)
                mbar_wait(vf0 + 8 * (uint32_t)(i % kVStages), (uint32_t)(i / kVStages) & 1u, err);
            if (qloads > 0) mbar_wait(qf, (uint32_t)(qloads - 1) & 1u, err);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------ MMA issuer (one thread)
        // Event loop: O(i) goes out as soon as P(i) is in, S(j) as soon as tile j has landed and
        // S buffer j % kSBufs is free (O(j - kSBufs), which reads the P there, has been issued:
        // the tcgen05 MMAs of one thread execute in issue order). No product waits behind a
        // later tile's load, and the loop polls two barriers per tile (each poll of shared
        // memory is slow while TMA and the tensor core stream through it). No tcgen05 fence
        // here: in this thread it would wait for the products in flight. The operands are
        // ordered by the mbarriers: TMA completion for K/V, and tcgen05.wait::st before every
        // arrival that hands over TMEM written by the softmax threads (P, a rescaled O).
        if (lane == 0) {
            const uint32_t idS = la_idesc(kRows, kTile, false), idO = la_idesc(kRows, kDh, true);
            LaCursor cs = la_cursor(s0, tab, lp), co = cs;
            int qwaits = 0;
            bool q_ready = false;  // the queries of S tile ns's run have landed
            int ns = 0, no = 0;  // next S tile, next O tile
            int run0 = 0;        // first local tile of the run the O products are in
            bool dead = false;
            uint64_t t_last = global_timer_ns();
            uint32_t spins = 0;
            while (no < n && !dead) {
                bool prog = false;
                // S buffer ns % kSBufs holds P(ns - kSBufs): S(ns) goes out after O(ns - kSBufs) has
                // been issued, and the MMAs of one thread execute in issue order
                if (ns < n && ns < no + kSBufs) {
                    const bool run_start = ns == 0 || cs.t == 0;
                    if (run_start && !q_ready && la_test_wait(qf, (uint32_t)qwaits & 1u)) {
                        q_ready = true;
                        ++qwaits;
                    }
                    const int sk = ns % kKStages;
                    if ((!run_start || q_ready) && la_test_wait(kf0 + 8 * sk, (uint32_t)(ns / kKStages) & 1u)) {
                        const uint32_t kb = sK + (uint32_t)sk * kOperand;
                        const uint32_t d = tmem + (uint32_t)(ns % kSBufs) * kTile;
#pragma unroll
                        for (int kk = 0; kk < kDh / 16; ++kk) {
                            const uint64_t a = la_desc(sQ + (uint32_t)(kk >> 2) * kQHalf + (uint32_t)(kk & 3) * 32, 16, 1024);
                            const uint64_t b = la_desc(kb + (uint32_t)(kk >> 2) * kHalf + (uint32_t)(kk & 3) * 32, 16, 1024);
                            la_mma(d, a, b, idS, kk > 0 ? 1u : 0u);
                        }
                        la_commit(sf0 + 8 * (uint32_t)(ns % kSBufs));
                        la_commit(ke0 + 8 * sk);  // K tile free once this S has completed
                        if (ns == n - 1 || cs.t == cs.nt - 1) la_commit(qe);  // the run's last S: Qd may go
                        q_ready = false;
                        ++ns;
                        if (ns < n) la_next(cs, tab, lp);
                        prog = true;
                    }
                }
                if (no < ns) {
                    const int sv = no % kVStages;
                    const uint32_t g = (uint32_t)(no & 1);
                    if (la_test_wait(pf0 + 8 * (uint32_t)(no % kSBufs), (uint32_t)(no / kSBufs) & 1u) &&
                        la_test_wait(vf0 + 8 * sv, (uint32_t)(no / kVStages) & 1u)) {
                        if (no == 0 || co.t == 0) run0 = no;
                        const bool first = no - run0 < 2;  // this group's first tile of the run: O afresh
                        // P(no) sits in the first 64 columns of S buffer no % kSBufs (bf16 pairs)
                        const uint32_t pa = tmem + (uint32_t)(no % kSBufs) * kTile;
                        const uint32_t vb = sV + (uint32_t)sv * kOperand;
#pragma unroll
                        for (int kk = 0; kk < kTile / 16; ++kk) {
                            const uint64_t b = la_desc(vb + (uint32_t)kk * 2048, kHalf, 1024);
                            la_mma_ts(tmem + kTmemO + g * kDh, pa + (uint32_t)kk * 8, b, idO, (!first || kk > 0) ? 1u : 0u);
                        }
                        la_commit(ve0 + 8 * sv);  // V tile free once this O has completed
                        la_commit(sx0 + 8 * (uint32_t)(no % kSBufs));
                        ++no;
                        la_next(co, tab, lp);
                        prog = true;
                    }
                }
                if (prog) {
                    spins = 0;
                    t_last = 0;
                } else if ((++spins & 255u) == 0u) {
                    // bounded: no progress for kWaitLimitNs (or 2^26 polls) gives up
                    const uint64_t now = global_timer_ns();
                    if (t_last == 0) t_last = now;
                    if (*(volatile int*)&s_abort || now - t_last > kWaitLimitNs || spins >= (1u << 26)) {
                        if (!*(volatile int*)&s_abort) set_error(err, kErrTimeout);
                        dead = true;
                    }
                }
            }
            if (dead) s_abort = 1;
            // every MMA issued has completed before TMEM is released
            la_commit(endb);
            mbar_wait(endb, 0, err);
        }
    } else {
        // ------------------------------------------------ softmax: two groups of 128 threads take
        // alternate tiles. Warp w of a group reads TMEM lane quarter w % 4, which holds rows
        // 16 (w % 4) .. 16 (w % 4) + 15 of the M = 64 accumulators; thread t of the warp owns rows
        // r0 = 16 (w % 4) + t/4 and r1 = r0 + 8 (window queries) and, of each 128-token tile, the
        // tokens 8j + 2 (t % 4) + {0, 1}, j = 0..15. The four threads of a quad share their rows:
        // the running max is the quad's, each thread sums the weights of its own tokens.
        const int g = warp >> 2, sp = warp & 3, cq = lane & 3;
        const int r0 = sp * 16 + (lane >> 2), r1 = r0 + 8;
        const uint32_t lane_t = tmem + ((uint32_t)(sp * 32) << 16);
        const uint32_t o0 = lane_t + kTmemO, o1 = o0 + kDh, o_mine = g ? o1 : o0;
        LaCursor cur = la_cursor(s0, tab, lp);
        bool anybad = false;
        if (lp.indexed) {
            // once per CTA: does any tile of its range hold an out-of-range id? Only then does each
            // tile build its bad-token mask (the ids' loads would otherwise sit in every tile's path)
            pdl_wait();  // the chunk ids come from the preceding kernel
            for (int64_t sidx = s0 + (tid & 255); sidx < s1; sidx += 256) {
                const LaCursor u = la_cursor(sidx, tab, lp);
                const int u0 = u.t * kTile;
                uint64_t bad = la_bad_tokens(u, u0, ids, tab);
                if (u.kt - u0 > kHalfTok) bad |= la_bad_tokens(u, u0 + kHalfTok, ids, tab);
                if (bad != 0ull) s_anybad = 1;
            }
            la_softmax_sync();
            anybad = *(volatile int*)&s_anybad != 0;
        }
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
        bool dead = false, run_whole = false;
        int run_idx = 0;
        int run0 = 0;
        for (int i = 0; i < n; ++i) {
            const bool last = (i == n - 1) || cur.t == cur.nt - 1;
            if (i == 0 || cur.t == 0) {
                m0 = m1 = -INFINITY;
                l0 = l1 = 0.f;
                run_whole = cur.t == 0;
                run0 = i;
            }
            if ((int)(i & 1) == g) {
                // valid tokens among this thread's 32 (bit 2j + e: token 8j + 2 cq + e of the tile):
                // inside the kept tokens and not from a chunk whose id is out of range
                uint32_t vm = 0xFFFFFFFFu;
                {
                    const int u0 = cur.t * kTile;
                    const int rem = cur.kt - u0;
                    uint64_t bad0 = 0ull, bad1 = 0ull;
                    if (anybad) {
                        bad0 = la_bad_tokens(cur, u0, ids, tab);
                        if (rem > kHalfTok) bad1 = la_bad_tokens(cur, u0 + kHalfTok, ids, tab);
                    }
                    if (rem < kTile || (bad0 | bad1) != 0ull) {
                        vm = 0u;
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const int tok = 8 * j + 2 * cq + e;
                                const uint64_t bw = tok < kHalfTok ? bad0 : bad1;
                                if (tok < rem && !((bw >> (tok & 63)) & 1ull)) vm |= 1u << (2 * j + e);
                            }
                        }
                    }
                }
                // 1. the scores of tile i: both 64-column halves in one TMEM round trip (the softmax
                // latency keeps the tile's V stage occupied, so it is on the ring's critical path)
                dead = la_wait_warp(dead, sf0 + 8 * (uint32_t)(i % kSBufs), (uint32_t)(i / kSBufs) & 1u, err,
                                    &s_abort);
                la_fence_after();
                const uint32_t sbuf = lane_t + (uint32_t)(i % kSBufs) * kTile;
                uint32_t sr[2][32];
                if (!dead) {
                    la_ld256x8(sbuf, sr[0]);
                    la_ld256x8(sbuf + 64u, sr[1]);
                    la_wait_ld();
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) sr[0][j] = sr[1][j] = 0u;
                }
                float mt0 = -INFINITY, mt1 = -INFINITY;
#pragma unroll
                for (int w = 0; w < 2; ++w) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int bit = 2 * (8 * w + j);
                        const bool v0 = (vm >> bit) & 1u, v1 = (vm >> (bit + 1)) & 1u;
                        mt0 = fmaxf(mt0, fmaxf(v0 ? __uint_as_float(sr[w][4 * j]) : -INFINITY,
                                               v1 ? __uint_as_float(sr[w][4 * j + 1]) : -INFINITY));
                        mt1 = fmaxf(mt1, fmaxf(v0 ? __uint_as_float(sr[w][4 * j + 2]) : -INFINITY,
                                               v1 ? __uint_as_float(sr[w][4 * j + 3]) : -INFINITY));
                    }
                }
                mt0 = fmaxf(mt0, __shfl_xor_sync(0xffffffffu, mt0, 1));
                mt0 = fmaxf(mt0, __shfl_xor_sync(0xffffffffu, mt0, 2));
                mt1 = fmaxf(mt1, __shfl_xor_sync(0xffffffffu, mt1, 1));
                mt1 = fmaxf(mt1, __shfl_xor_sync(0xffffffffu, mt1, 2));
                mt0 *= lp.qscale;
                mt1 *= lp.qscale;
                // 2. running max (log2 domain); a row's O is rescaled only when its max grows past 2^8
                const float mn0 = fmaxf(m0, mt0), mn1 = fmaxf(m1, mt1);
                float a0 = 1.f, a1 = 1.f;
                bool need = false;
                if (i - run0 < 2) {
                    m0 = mn0;  // this group's first tile of the run: O starts afresh
                    m1 = mn1;
                } else {
                    if (mn0 > m0 + kRescale) {
                        need = true;
                        a0 = la_ex2(m0 - mn0);
                        m0 = mn0;
                    }
                    if (mn1 > m1 + kRescale) {
                        need = true;
                        a1 = la_ex2(m1 - mn1);
                        m1 = mn1;
                    }
                }
                if (__any_sync(0xffffffffu, need)) {
                    // the group's previous O product (tile i - 2) has finished: its O rows are stable.
                    // (Waited on the per-buffer barrier: S(i) has landed, so O(i - 4) is done and the
                    // phase awaited is the pending one or the last completed, never two ahead.)
                    dead = la_wait_warp(dead, sx0 + 8 * (uint32_t)((i - 2) % kSBufs), (uint32_t)((i - 2) / kSBufs) & 1u,
                                        err, &s_abort);
                    la_fence_after();
                    if (!dead) {
#pragma unroll 1
                        for (int w = 0; w < 2; ++w) {
                            uint32_t o[32];
                            la_ld256x8(o_mine + (uint32_t)(w * 64), o);
                            la_wait_ld();
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                o[4 * j] = __float_as_uint(__uint_as_float(o[4 * j]) * a0);
                                o[4 * j + 1] = __float_as_uint(__uint_as_float(o[4 * j + 1]) * a0);
                                o[4 * j + 2] = __float_as_uint(__uint_as_float(o[4 * j + 2]) * a1);
                                o[4 * j + 3] = __float_as_uint(__uint_as_float(o[4 * j + 3]) * a1);
                            }
                            la_st256x8(o_mine + (uint32_t)(w * 64), o);
                        }
                        la_wait_st();
                    }
                    l0 *= a0;
                    l1 *= a1;
                }
                // 3. P = 2^(s c - m) as bf16 pairs over the first 64 columns of this S buffer: the
                // pair of tokens 64w + 8j + 2cq + {0, 1} goes to column 32w + 4j + cq (the scores are
                // all in registers already). l sums the fp32 weights.
                const float nm0 = m0 == -INFINITY ? 0.f : -m0;  // all masked so far: every p is 0
                const float nm1 = m1 == -INFINITY ? 0.f : -m1;
                float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
                for (int w = 0; w < 2; ++w) {
                    uint32_t pk[16];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int bit = 2 * (8 * w + j);
                        const bool v0 = (vm >> bit) & 1u, v1 = (vm >> (bit + 1)) & 1u;
                        const float p00 = v0 ? la_ex2(fmaf(__uint_as_float(sr[w][4 * j]), lp.qscale, nm0)) : 0.f;
                        const float p01 = v1 ? la_ex2(fmaf(__uint_as_float(sr[w][4 * j + 1]), lp.qscale, nm0)) : 0.f;
                        const float p10 = v0 ? la_ex2(fmaf(__uint_as_float(sr[w][4 * j + 2]), lp.qscale, nm1)) : 0.f;
                        const float p11 = v1 ? la_ex2(fmaf(__uint_as_float(sr[w][4 * j + 3]), lp.qscale, nm1)) : 0.f;
                        ps0 += p00 + p01;
                        ps1 += p10 + p11;
                        const __nv_bfloat162 h0 = __floats2bfloat162_rn(p00, p01);
                        const __nv_bfloat162 h1 = __floats2bfloat162_rn(p10, p11);
                        pk[2 * j] = *reinterpret_cast<const uint32_t*>(&h0);
                        pk[2 * j + 1] = *reinterpret_cast<const uint32_t*>(&h1);
                    }
                    if (!dead) la_st128x8(sbuf + (uint32_t)(w * 32), pk);
                }
                l0 += ps0;
                l1 += ps1;
                if (!dead) la_wait_st();
                la_fence_before();
                mbar_arrive(pf0 + 8 * (uint32_t)(i % kSBufs));
            }

            // 4. end of this CTA's part of run (b, h): merge the two groups' rows (same TMEM lanes,
            // different columns), then write out (whole run) or a partial (run split across CTAs)
            if (last) {
                const int jl = ((i & 1) == g) ? i : i - 1;  // this group's last tile of the run
                if (jl >= run0)
                    dead = la_wait_warp(dead, sx0 + 8 * (uint32_t)(jl % kSBufs), (uint32_t)(jl / kSBufs) & 1u, err,
                                        &s_abort);
                // each row's sum: the quad's four parts
                float L0 = l0 + __shfl_xor_sync(0xffffffffu, l0, 1);
                L0 += __shfl_xor_sync(0xffffffffu, L0, 2);
                float L1 = l1 + __shfl_xor_sync(0xffffffffu, l1, 1);
                L1 += __shfl_xor_sync(0xffffffffu, L1, 2);
                if (g == 1 && cq == 0) {
                    s_ml1[r0] = make_float2(m0, L0);
                    s_ml1[r1] = make_float2(m1, L1);
                }
                la_fence_before();
                la_softmax_sync();  // group 1's last O has completed and its (m, l) are in s_ml1
                la_fence_after();
                if (g == 0) {
                    const float2 b0 = s_ml1[r0], b1 = s_ml1[r1];
                    const float M0 = fmaxf(m0, b0.x), M1 = fmaxf(m1, b1.x);
                    // a group that took no tile of the run has m = -inf: weight 0, its O is not read
                    const float w00 = m0 == -INFINITY ? 0.f : la_ex2(m0 - M0);
                    const float w01 = b0.x == -INFINITY ? 0.f : la_ex2(b0.x - M0);
                    const float w10 = m1 == -INFINITY ? 0.f : la_ex2(m1 - M1);
                    const float w11 = b1.x == -INFINITY ? 0.f : la_ex2(b1.x - M1);
                    const float LL0 = w00 * L0 + w01 * b0.y, LL1 = w10 * L1 + w11 * b1.y;
                    const bool whole = run_whole && cur.t == cur.nt - 1;
                    const bool wr0 = r0 < lp.Qw && !dead, wr1 = r1 < lp.Qw && !dead;
                    const int64_t slot = 2 * (int64_t)c + (run_idx == 0 ? 0 : 1);
                    float* dst0 = whole ? out + (((int64_t)cur.b * lp.Qw + r0) * lp.H + cur.h) * kDh
                                        : part_o + (slot * lp.Qw + r0) * kDh;
                    float* dst1 = whole ? out + (((int64_t)cur.b * lp.Qw + r1) * lp.H + cur.h) * kDh
                                        : part_o + (slot * lp.Qw + r1) * kDh;
                    // no valid token at all (every id bad): out 0, lse -inf
                    const float inv0 = whole ? (LL0 > 0.f ? 1.f / LL0 : 0.f) : 1.f;
                    const float inv1 = whole ? (LL1 > 0.f ? 1.f / LL1 : 0.f) : 1.f;
#pragma unroll 1
                    for (int w = 0; w < 2; ++w) {
                        uint32_t oa[32], ob[32];
                        if (!dead) {
                            la_ld256x8(o0 + (uint32_t)(w * 64), oa);
                            la_ld256x8(o1 + (uint32_t)(w * 64), ob);
                            la_wait_ld();
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j) oa[j] = ob[j] = 0u;
                        }
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const int col = 64 * w + 8 * j + 2 * cq;
                            float x[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float wa = e < 2 ? w00 : w10, wb = e < 2 ? w01 : w11;
                                float v = wa != 0.f ? wa * __uint_as_float(oa[4 * j + e]) : 0.f;
                                if (wb != 0.f) v = fmaf(wb, __uint_as_float(ob[4 * j + e]), v);
                                x[e] = v * (e < 2 ? inv0 : inv1);
                            }
                            if (wr0) *reinterpret_cast<float2*>(dst0 + col) = make_float2(x[0], x[1]);
                            if (wr1) *reinterpret_cast<float2*>(dst1 + col) = make_float2(x[2], x[3]);
                        }
                    }
                    if (cq == 0) {
                        if (whole) {
                            if (lse != nullptr) {
                                if (wr0) lse[((int64_t)cur.b * lp.Qw + r0) * lp.H + cur.h] = (M0 + log2f(LL0)) * kLn2;
                                if (wr1) lse[((int64_t)cur.b * lp.Qw + r1) * lp.H + cur.h] = (M1 + log2f(LL1)) * kLn2;
                            }
                        } else {
                            if (wr0) *reinterpret_cast<float2*>(part_ml + (slot * lp.Qw + r0) * 2) = make_float2(M0, LL0);
                            if (wr1) *reinterpret_cast<float2*>(part_ml + (slot * lp.Qw + r1) * 2) = make_float2(M1, LL1);
                        }
                    }
                }
                la_softmax_sync();  // s_ml1 is read before a later run end writes it again
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

// Merge of the partials of the runs split across CTAs (log-sum-exp rule). grid (B*H, ceil(Qw/4)),
// 128 threads: warp w merges window query blockIdx.y*4 + w; lane k owns output columns 4k..4k+3.
// 128-thread CTAs fit on an SM beside a k_attn_la CTA (registers), so they are resident and
// waiting when the attention grid completes.
constexpr int kLaMergeWarps = 4;
__global__ void __launch_bounds__(kLaMergeWarps * 32)
k_attn_la_merge(const float* __restrict__ part_o, const float* __restrict__ part_ml, float* __restrict__ out,
                float* __restrict__ lse, const SeqTable tab, const LaParams lp) {
    const int g = blockIdx.x, b = g / lp.H, h = g - b * lp.H;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = blockIdx.y * kLaMergeWarps + w;
    pdl_trigger();  // the next kernel may set itself up; its reads wait for this grid
    pdl_wait();
    if (q >= lp.Qw) return;
    const int kt = (tab.kept_off[b + 1] - tab.kept_off[b]) * tab.C;
    const int nt = (kt + la::kTile - 1) / la::kTile;
    const int64_t ts = lp.tile_off[b] + (int64_t)h * nt, te = ts + nt;
    const int c0 = la_cta_of(ts, lp), c1 = la_cta_of(te - 1, lp);
    if (c0 == c1) return;  // written directly by its CTA
    const int ns = c1 - c0 + 1;
    // the run is the first run of every CTA after c0; of c0 only if c0's tiles start inside it
    const int slot0 = 2 * c0 + (lp.cta_start[c0] == ts ? 0 : 1);
    auto slot_of = [&](int i) { return i == 0 ? slot0 : 2 * (c0 + i); };

    // chunks of up to 16 pieces, each one round trip: lane i loads (m, l) of piece i of the chunk
    // while every lane loads its 4 columns of all the chunk's rows; the running max rescales
    float M = -INFINITY, L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    constexpr int kU = 16;  // partial rows in flight per lane
    for (int i0 = 0; i0 < ns; i0 += kU) {
        const int cnt = ns - i0 < kU ? ns - i0 : kU;
        float2 ml = make_float2(-INFINITY, 0.f);
        if (lane < cnt) ml = *reinterpret_cast<const float2*>(part_ml + ((int64_t)slot_of(i0 + lane) * lp.Qw + q) * 2);
        float4 v[kU];  // rows past the chunk reload its last row (weight 0), so every load is issued
#pragma unroll
        for (int u = 0; u < kU; ++u)
            v[u] = *reinterpret_cast<const float4*>(
                part_o + ((int64_t)slot_of(i0 + (u < cnt ? u : cnt - 1)) * lp.Qw + q) * kDh + lane * 4);
        float mc = ml.x;
        for (int off = 16; off > 0; off >>= 1) mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, off));
        const float Mn = fmaxf(M, mc);
        const float a = M == -INFINITY ? 0.f : la_ex2(M - Mn);  // rescale of the earlier chunks
        const float wgt = ml.x == -INFINITY ? 0.f : la_ex2(ml.x - Mn);
        float lc = wgt * ml.y;
        for (int off = 16; off > 0; off >>= 1) lc += __shfl_xor_sync(0xffffffffu, lc, off);
        L = fmaf(L, a, lc);
        acc = make_float4(acc.x * a, acc.y * a, acc.z * a, acc.w * a);
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const float wj = u < cnt ? __shfl_sync(0xffffffffu, wgt, u) : 0.f;
            acc.x = fmaf(wj, v[u].x, acc.x);
            acc.y = fmaf(wj, v[u].y, acc.y);
            acc.z = fmaf(wj, v[u].z, acc.z);
            acc.w = fmaf(wj, v[u].w, acc.w);
        }
        M = Mn;
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;  // no valid token (every id bad): out 0, lse -inf
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

// Tiles of one (sequence, head) run of kt kept tokens.
static int64_t la_run_tiles(int64_t kt) { return (kt + la::kTile - 1) / la::kTile; }

// Tiles of the global list (sum over sequences of H * ceil(k_b * C / 128)).
int64_t la_tiles(const lsa_dims& d, const SeqTable& tab) {
    int64_t S = 0;
    for (int b = 0; b < d.B; ++b)
        S += (int64_t)d.H * la_run_tiles((int64_t)(tab.kept_off[b + 1] - tab.kept_off[b]) * tab.C);
    return S;
}

// Split of the global tile list over the CTAs, by cost rather than by count: a tile costs 1
// and the start of a (sequence, head) run W more (its query reload and run-end merge take about
// as long as W tiles), so a CTA that opens a run takes fewer tiles. cost(s) = s + W * run(s)
// increases with s; CTA c takes the tiles with ceil(c F / G) <= cost < ceil((c + 1) F / G),
// F = S + W (runs - 1), one contiguous range each. A split that would leave a CTA empty (short
// lists) falls back to the even split (W = 0). Writes cta_start[0..G] and returns G.
int la_partition(const SeqTable& tab, int H, int max_ctas, int32_t* cta_start) {
    int64_t S = 0;
    for (int b = 0; b < tab.B; ++b)
        S += (int64_t)H * la_run_tiles((int64_t)(tab.kept_off[b + 1] - tab.kept_off[b]) * tab.C);
    int G = (int)(S < max_ctas ? S : max_ctas);
    if (G > la::kMaxCtas) G = la::kMaxCtas;
    const int64_t runs = (int64_t)tab.B * H;
    for (int W = la::kRunCost; W >= 0; W -= la::kRunCost) {
        const int64_t F = S + W * (runs - 1);
        int b = 0;
        int64_t off = 0;  // first tile of sequence b
        for (int c = 0; c <= G; ++c) {
            const int64_t T = (c * F + G - 1) / G;  // least cost of CTA c
            int64_t s = S;
            for (; b < tab.B; ++b) {
                const int64_t nt = la_run_tiles((int64_t)(tab.kept_off[b + 1] - tab.kept_off[b]) * tab.C);
                const int64_t base = off + W * (int64_t)b * H;  // cost of the sequence's first tile
                const int64_t last = base + (H - 1) * (nt + W) + nt - 1;
                if (T <= last) {
                    if (T <= base) {
                        s = off;
                    } else {
                        const int64_t h = (T - base) / (nt + W), t = T - base - h * (nt + W);
                        s = t < nt ? off + h * nt + t : off + (h + 1) * nt;
                    }
                    break;
                }
                off += (int64_t)H * nt;
            }
            cta_start[c] = (int32_t)s;
        }
        bool ok = true;
        for (int c = 0; c < G; ++c) ok = ok && cta_start[c] < cta_start[c + 1];
        if (ok || W == 0) break;
    }
    return G;
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
    lp.G = la_partition(tab, d.H, max_ctas, lp.cta_start);
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
    mc.gridDim = dim3(d.B * d.H, (d.Q + kLaMergeWarps - 1) / kLaMergeWarps, 1);
    mc.blockDim = dim3(kLaMergeWarps * 32, 1, 1);
    mc.dynamicSmemBytes = 0;
    const float* cpo = part_o;
    const float* cpm = part_ml;
    return cudaLaunchKernelEx(&mc, k_attn_la_merge, cpo, cpm, out, lse, tab, lp);
}

}  // namespace lsa
