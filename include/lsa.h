/*
 * lsa.h - C ABI of the Lookahead Sparse Attention (LSA) decode step, B200 (sm_100a).
 *
 * The method (FlashMemory-DeepSeek-V4, "Lightning Index Ultra-Long Context via
 * Lookahead Sparse Attention", arXiv 2606.09079): at a decode step a dual-encoder
 * Neural Memory Indexer scores every historical KV chunk against the query side,
 * a top-k keep mask keeps the query-critical chunks, and decode attention runs
 * over the kept chunks only. Sources, by page and section:
 *   [R3-2.1] dimensionstp.github.io review, section 3-2 (1): the KV cache is
 *            treated as chunk-granular memory (the cache unit is a chunk);
 *   [R3-2.2] same review, section 3-2 (2) "Neural Memory Indexer": chunk
 *            relevance scoring; layer scores are combined with a max;
 *   [R3-2.3] same review, section 3-2 (3) "Lookahead Sparse Attention",
 *            steps 4-7: score all chunks, top-k keep mask, attend over the kept
 *            chunks only; the lookahead window is about 64 tokens;
 *   [ABS]    the arXiv abstract: the indexer is a standard dual encoder (so a
 *            relevance score is an inner product) and only the query-critical
 *            KV chunks stay resident in GPU memory.
 *
 * Conventions for every call
 *   - All tensor pointers are DEVICE pointers owned by the caller, 16-byte
 *     aligned, row-major and contiguous. The library never allocates or frees
 *     memory and never synchronises, except lsa_get_device_status.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL is the legacy default stream). Calls can be captured in a CUDA graph.
 *   - Arguments are validated on the host before anything is launched; a bad
 *     argument returns LSA_ERR_INVALID_ARG / LSA_ERR_UNSUPPORTED / LSA_ERR_WORKSPACE
 *     and launches nothing. A launch failure returns LSA_ERR_CUDA.
 *   - Errors found on the device (a non-finite score, a kept chunk id out of
 *     range, a bounded wait that gave up) set bits of a sticky error word at the
 *     start of the workspace; the kernels then skip the bad item instead of
 *     faulting. lsa_get_device_status reads and clears that word.
 *   - Per-device facts (SM count, kernel attributes) are looked up on the first
 *     call made on a device and cached for the life of the process; the library
 *     is not meant to be used across a cudaDeviceReset.
 *   - Ragged batches: with chunk_offsets != NULL, sequence b owns chunks
 *     [chunk_offsets[b], chunk_offsets[b+1]) of the flattened chunk axis and
 *     tokens [chunk_offsets[b]*C, chunk_offsets[b+1]*C) of the K/V caches.
 *     Kept ids are laid out flat: sequence b's k_b ids start at sum_{b'<b} k_b'.
 */
#ifndef LSA_H_
#define LSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define LSA_API __attribute__((visibility("default")))
#else
#define LSA_API
#endif

#define LSA_ABI_VERSION 1
#define LSA_MAX_BATCH 256   /* sequences per call */
#define LSA_HEAD_DIM 128    /* Dh: the pages' HEAD_DIM (review, section 4-3) */
#define LSA_INDEX_DIM 128   /* compressed-K key dim: 128 e4m3 values per 132-byte chunk (review, section 3-2 (1)) */

typedef enum {
    LSA_OK = 0,
    LSA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size, k outside 1..N_b */
    LSA_ERR_WORKSPACE = 2,    /* workspace smaller than lsa_workspace_size() */
    LSA_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
    LSA_ERR_NONFINITE = 4,    /* device: a chunk score was NaN or +-Inf */
    LSA_ERR_TIMEOUT = 5,      /* device: a bounded wait gave up */
    LSA_ERR_UNSUPPORTED = 6,  /* a shape the library does not implement */
    LSA_ERR_BAD_ID = 7        /* device: a kept chunk id was outside 0..N_b-1 */
} lsa_status;

typedef enum { LSA_F32 = 0, LSA_BF16 = 1 } lsa_dtype;

/* How the per-layer indexer scores are combined (review, section 3-2 (2): max or mean). */
typedef enum { LSA_ENSEMBLE_MAX = 0, LSA_ENSEMBLE_MEAN = 1 } lsa_ensemble;

/* Problem shape of one call. Host memory; copied by value into the launch. */
typedef struct {
    int32_t B;          /* sequences, 1..LSA_MAX_BATCH */
    int32_t Q;          /* query embeddings per sequence: 1 (decode query) .. 256 (64 = lookahead window) */
    int32_t E;          /* embedding dim; E*sizeof(emb) a power of two in 16..512 bytes, or a multiple of 512 */
    int32_t H;          /* attention heads (query heads = KV heads), a power of two, 1..128 */
    int32_t Dh;         /* head dim, must be LSA_HEAD_DIM */
    int32_t chunk_len;  /* C, tokens per chunk, a power of two, 8..1024 (64 in the workloads) */
    int32_t N;          /* chunks per sequence when chunk_offsets == NULL */
    int32_t k;          /* kept chunks per sequence when k_per_seq == NULL */
    const int64_t *chunk_offsets; /* host [B+1], nondecreasing from 0, or NULL (uniform N) */
    const int32_t *k_per_seq;     /* host [B], or NULL (uniform k) */
    lsa_dtype emb_dtype;          /* q_emb and chunk_emb */
    lsa_dtype kv_dtype;           /* q, K, V, K_res, V_res */
} lsa_dims;

/* ABI version of the loaded library (LSA_ABI_VERSION). */
LSA_API int lsa_abi_version(void);

/* Human-readable name of a status code (static string). */
LSA_API const char *lsa_status_string(lsa_status s);

/* Bytes of device workspace the calls below need for `dims` on the current
 * device (it depends on the SM count). Writes *bytes; no launch. */
LSA_API lsa_status lsa_workspace_size(const lsa_dims *dims, size_t *bytes);

/* Clear the workspace header (cudaMemsetAsync of its first 256 bytes): the sticky
 * error word and the arrival counters of the one-launch step, which every such step
 * leaves at zero again. Call once after allocating a workspace. */
LSA_API lsa_status lsa_workspace_init(void *ws, size_t ws_bytes, void *stream);

/* Chunk relevance [R3-2.2, ABS, R3-2.3 step 4].
 *   q_emb     [B][Q][E]      emb_dtype
 *   chunk_emb [sum N_b][E]   emb_dtype
 *   scores    [sum N_b]      float32, out:  scores[i] = max_j <q_emb[b][j], chunk_emb[i]>
 * fp32 accumulation. Q == 1 streams the embeddings on CUDA cores; Q > 1 with bf16
 * embeddings and E <= 256 runs a tcgen05 tensor-core GEMM with a per-row max. */
LSA_API lsa_status lsa_score_chunks(const lsa_dims *dims, const void *q_emb, const void *chunk_emb,
                            float *scores, void *ws, size_t ws_bytes, void *stream);

/* The Neural Memory Indexer's score on FP8 compressed-K chunks [R3-2.2; review sections
 * 3-2 (1) (the 132-byte chunk format) and 4-3 (128 heads x 128 dims)]:
 *   s_i = ensemble_l sigmoid( sum_h w_lh * ReLU( ks_li * qs_blh * (q8_blh . k8_li) ) )
 *   compressed_k [L][sum N_b][132] bytes: 128 float8_e4m3 key values, then the float32
 *                dequant scale ks (little-endian), per layer and chunk
 *   q_fp8        [B][L][n_heads][128] float8_e4m3 queries (the query-side projection, norm,
 *                RoPE and Hadamard transform happen before this call)
 *   q_scale      [B][L][n_heads] float32 query dequant scales;  head_w [L][n_heads] float32
 *   scores       [sum N_b] float32, out
 * dims->E must be LSA_INDEX_DIM; n_layers 1..16; n_heads a multiple of 16 in 16..256.
 * A tcgen05 kind::f8f6f4 tensor-core GEMM (e4m3 x e4m3 -> fp32 in TMEM) per layer. */
LSA_API lsa_status lsa_indexer_score_fp8(const lsa_dims *dims, int32_t n_layers, int32_t n_heads,
                                         lsa_ensemble ensemble, const void *compressed_k, const void *q_fp8,
                                         const float *q_scale, const float *head_w, float *scores, void *ws,
                                         size_t ws_bytes, void *stream);

/* Top-k keep mask [R3-2.3 step 5].
 *   scores    [sum N_b]   float32
 *   chunk_ids [sum k_b]   int32, out: per sequence the k_b chunk indices (0..N_b-1,
 *                         local to the sequence) with the highest scores, ties to the
 *                         lower index, written in ascending order. -0.0 == +0.0.
 * A NaN/Inf score sets LSA_ERR_NONFINITE in the sticky word (ids stay in range). */
LSA_API lsa_status lsa_topk_select(const lsa_dims *dims, const float *scores, int32_t *chunk_ids,
                           void *ws, size_t ws_bytes, void *stream);

/* Threshold keep mask with a fallback floor [R3-2.3 step 5: "top-k or threshold";
 * review section 4-3: precise-needle tasks need a threshold fallback]. The pages give no
 * rule; this library's: k_eff = clamp(#{i : s_i >= tau}, min(k_min, k_b), k_b) and the kept
 * set is the top-k_eff by (score desc, index asc), so the fallback keeps at least k_min chunks
 * and the capacity k_b (dims k / k_per_seq) caps the count.
 *   scores     [sum N_b] float32;  tau finite; k_min >= 1
 *   chunk_ids  [sum k_b] int32, out: per sequence the k_eff kept ids ascending, then -1
 *   kept_count [B] int32 device, out: k_eff per sequence. */
LSA_API lsa_status lsa_threshold_select(const lsa_dims *dims, const float *scores, float tau, int32_t k_min,
                                        int32_t *chunk_ids, int32_t *kept_count, void *ws, size_t ws_bytes,
                                        void *stream);

/* Gather of the kept chunks into a compact resident buffer [R3-2.3 step 6, ABS].
 *   K, V         [sum L_b][H][Dh]   kv_dtype (L_b = N_b * C)
 *   chunk_ids    [sum k_b]          int32, local chunk indices
 *   K_res, V_res [sum k_b * C][H][Dh] kv_dtype, out: row j*C+t of sequence b's
 *                block is row ids[j]*C+t of its cache.
 * An id outside 0..N_b-1 sets LSA_ERR_BAD_ID and that chunk is left unwritten. */
LSA_API lsa_status lsa_gather_kv(const lsa_dims *dims, const void *K, const void *V,
                         const int32_t *chunk_ids, void *K_res, void *V_res,
                         void *ws, size_t ws_bytes, void *stream);

/* Sparse decode attention over the kept tokens [R3-2.3 steps 6-7].
 *   q         [B][H][Dh]  kv_dtype, one decode query per sequence
 *   K, V      chunk_ids != NULL: the full caches [sum L_b][H][Dh], read through the ids;
 *             chunk_ids == NULL: resident buffers [sum k_b*C][H][Dh] (lsa_gather_kv output)
 *   out       [B][H][Dh]  float32: softmax(q.K^T / sqrt(Dh)) V over the kept tokens
 *   lse       [B][H]      float32 natural-log sum of exp of the scaled logits, or NULL
 * Split-K flash-decode with fp32 online softmax and a log-sum-exp merge. */
LSA_API lsa_status lsa_sparse_decode_attn(const lsa_dims *dims, const void *q, const void *K,
                                  const void *V, const int32_t *chunk_ids, float *out,
                                  float *lse, void *ws, size_t ws_bytes, void *stream);

/* The fused step: score -> top-k -> attention over the kept chunks, reading K/V
 * through the kept ids (no resident copy is materialised) [R3-2.3 steps 4-7].
 * Arguments as above; chunk_ids_out [sum k_b] receives the kept ids; the scores
 * live in the workspace. Four kernels chained with programmatic dependent launch;
 * small problems (Q == 1, B*H <= 48, N_b <= 256, embedding rows <= 512 bytes, kept
 * K/V <= 16 MiB) run all four steps in one launch instead, whose arrival counters
 * live in the workspace header: the workspace must have been initialised with
 * lsa_workspace_init, and calls sharing a workspace must not overlap on the GPU. */
LSA_API lsa_status lsa_decode_step(const lsa_dims *dims, const void *q_emb, const void *chunk_emb,
                           const void *q, const void *K, const void *V,
                           int32_t *chunk_ids_out, float *out, float *lse,
                           void *ws, size_t ws_bytes, void *stream);

/* Attention of every query of the lookahead window over the kept tokens [R3-2.3: the indexer
 * keeps the chunks that the next ~64 tokens will attend to; steps 6-7]. Each of the
 * dims->Q window queries is an independent decode query over the same kept set, with no
 * mask between the window's queries:
 *   q         [B][Q][H][Dh] bf16, the window's attention queries (Q = dims->Q, 1..64)
 *   K, V      bf16; chunk_ids != NULL: the full caches [sum L_b][H][Dh] read through the ids;
 *             chunk_ids == NULL: resident buffers [sum k_b*C][H][Dh]
 *   out       [B][Q][H][Dh] float32: softmax(q_j . K^T / sqrt(Dh)) V over the kept tokens
 *   lse       [B][Q][H] float32 natural-log sums, or NULL
 * kv_dtype must be LSA_BF16 and Q <= 64 (else LSA_ERR_UNSUPPORTED); the token rows of K/V
 * must number below 2^31. A tcgen05 flash-attention kernel: S = Q.K^T and O += P.V on the
 * tensor cores (bf16 operands, fp32 accumulation, P rounded to bf16), online softmax in fp32,
 * split-K over one SM-balanced tile list with a log-sum-exp merge. */
LSA_API lsa_status lsa_sparse_decode_attn_lookahead(const lsa_dims *dims, const void *q, const void *K,
                                                    const void *V, const int32_t *chunk_ids, float *out,
                                                    float *lse, void *ws, size_t ws_bytes, void *stream);

/* The fused lookahead step: score with the window's Q query embeddings (max over them) ->
 * top-k -> every window query's attention over the kept chunks [R3-2.3 steps 4-7].
 * q_emb [B][Q][E]; q [B][Q][H][Dh] bf16; other arguments as lsa_decode_step and
 * lsa_sparse_decode_attn_lookahead. Four kernels chained with programmatic dependent launch. */
LSA_API lsa_status lsa_decode_step_lookahead(const lsa_dims *dims, const void *q_emb, const void *chunk_emb,
                                             const void *q, const void *K, const void *V,
                                             int32_t *chunk_ids_out, float *out, float *lse, void *ws,
                                             size_t ws_bytes, void *stream);

/* The split of the lookahead attention's tile list over its CTAs, exactly as
 * lsa_sparse_decode_attn_lookahead uses it. Host only: no device call, no GPU needed. This is
 * not an operation of the method (the pages define none like it): it exposes how this library
 * schedules the window attention [R3-2.3 steps 6-7], for tests and for callers sizing work.
 * The list holds, for each sequence b and then each head h, ceil(k_b * C / 128) tiles of
 * 128 kept tokens (one (sequence, head) run). A tile costs 1 and the start of a run 4 more;
 * CTA c takes the contiguous tiles whose cost lies in [ceil(c*F/G), ceil((c+1)*F/G)), with
 * F the total cost and G = min(tiles, max_ctas, 256). Where that would leave a CTA without
 * tiles, every tile costs 1 (the even split).
 *   max_ctas   CTAs to split over (the attention launches one per SM), >= 1
 *   cta_start  host array of at least min(max_ctas, 256) + 1 int32: the first tile of each
 *              CTA, then cta_start[G] = the number of tiles
 *   n_ctas     host int32, receives G
 * Errors: LSA_ERR_INVALID_ARG (bad dims, null pointer, max_ctas < 1), LSA_ERR_UNSUPPORTED
 * (a shape the lookahead attention does not take). */
LSA_API lsa_status lsa_lookahead_partition(const lsa_dims *dims, int32_t max_ctas, int32_t *cta_start,
                                           int32_t *n_ctas);

/* Retrieval cycle of the lookahead loop [R3-2.3 steps 4-7; review section 3-1: the
 * indexer re-scores about every 64 decode steps and attention runs over the kept
 * chunks until the next cycle]. Scores every chunk, keeps the top-k, and refreshes a
 * resident buffer so that it holds exactly the kept chunks, copying only entering ones.
 *   slot_ids     [sum k_b] int32, in/out: slot j of sequence b holds local chunk
 *                slot_ids[kept_off_b + j], or is empty (-1; fill with -1 for a cold start).
 *                Chunks that stay keep their slot; entering chunks (ascending) fill the freed
 *                slots (ascending). A chunk listed twice stays in one of its slots only.
 *   K_res, V_res [sum k_b * C][H][Dh] kv_dtype, in/out: slot j = rows [(kept_off_b+j)*C, +C).
 *   moved        [B] int32 device, out, or NULL: chunks copied per sequence.
 * Per-step attention between cycles: lsa_sparse_decode_attn with chunk_ids = NULL over
 * K_res/V_res (the slot order does not change the softmax). Requires N_b <= 2^19. */
LSA_API lsa_status lsa_refresh_resident(const lsa_dims *dims, const void *q_emb, const void *chunk_emb,
                                        const void *K, const void *V, int32_t *slot_ids, void *K_res,
                                        void *V_res, int32_t *moved, void *ws, size_t ws_bytes,
                                        void *stream);

/* Sparse decode attention for callers that cannot allocate device memory.
 * The paper has no counterpart: this is a deployment variant of
 * lsa_sparse_decode_attn for callers that cannot call cudaMalloc (an engine that
 * has reserved nearly all device memory for its own pool, a plugin that must not
 * allocate behind its host framework's allocator, or a latency-critical path where
 * cudaMalloc's implicit device synchronisation is not acceptable).
 * Arguments and results are those of lsa_sparse_decode_attn, without a workspace:
 * the split-K partials live in a fixed LSA_NOALLOC_SCRATCH_BYTES array inside the
 * library (allocated once per GPU that loads the library, held until exit).
 *   - Shapes whose partials, (device CTAs + B) * H * (Dh + 2) * 4 bytes plus 256,
 *     exceed that size are rejected with LSA_ERR_WORKSPACE before any launch.
 *   - It calls no allocation routine of any kind.
 *   - The first call on a device (with that device current) looks up the array's
 *     device address and the device's SM count; make that first call before any
 *     stream capture. Both are cached per process and per device ordinal for the
 *     life of the process: after cudaDeviceReset (a new primary context) the cached
 *     address names an array that no longer exists, so do not use this entry point
 *     across a device reset.
 *   - All calls on a device share the array, which keeps the last call's contents;
 *     each call clears the device error word it uses. Calls whose kernels overlap
 *     on the GPU race on the array: order them on one stream.
 *   - Device-side errors (a kept chunk id out of range) are skipped without a fault
 *     but are not reported: the error word is internal to the library. */
#define LSA_NOALLOC_SCRATCH_BYTES (4u << 20)
LSA_API lsa_status lsa_sparse_decode_attn_noalloc(const lsa_dims *dims, const void *q, const void *K,
                                                  const void *V, const int32_t *chunk_ids, float *out,
                                                  float *lse, void *stream);

/* The fused step with the threshold keep mask: score -> threshold select (as
 * lsa_threshold_select) -> attention over each sequence's k_eff kept chunks (read through
 * the ids; positions past kept_count are skipped on the device, so the host never waits).
 * Outputs as lsa_decode_step plus kept_count_out [B] int32 device. */
LSA_API lsa_status lsa_decode_step_threshold(const lsa_dims *dims, const void *q_emb, const void *chunk_emb,
                                             const void *q, const void *K, const void *V, float tau,
                                             int32_t k_min, int32_t *chunk_ids_out, int32_t *kept_count_out,
                                             float *out, float *lse, void *ws, size_t ws_bytes, void *stream);

/* The fused step with the FP8 indexer score: lsa_indexer_score_fp8 -> top-k -> attention
 * over the kept chunks (as lsa_decode_step, whose q_emb/chunk_emb are replaced by the
 * indexer inputs). */
LSA_API lsa_status lsa_decode_step_fp8(const lsa_dims *dims, int32_t n_layers, int32_t n_heads,
                                       lsa_ensemble ensemble, const void *compressed_k, const void *q_fp8,
                                       const float *q_scale, const float *head_w, const void *q, const void *K,
                                       const void *V, int32_t *chunk_ids_out, float *out, float *lse, void *ws,
                                       size_t ws_bytes, void *stream);

/* Sparse decode attention over a per-sequence device count of kept chunks: as
 * lsa_sparse_decode_attn with chunk_ids (the capacity k_b from dims), attending over the
 * first kept_count[b] ids only (kept_count [B] int32 device, 0 <= count <= k_b). A count of 0
 * gives out = 0 and lse = -inf. */
LSA_API lsa_status lsa_sparse_decode_attn_counts(const lsa_dims *dims, const void *q, const void *K,
                                                 const void *V, const int32_t *chunk_ids,
                                                 const int32_t *kept_count, float *out, float *lse, void *ws,
                                                 size_t ws_bytes, void *stream);

/* Chunk-sharded step across G ranks (this library's multi-GPU form of [R3-2.3 steps 4-7]:
 * a sequence's chunks are split into contiguous runs, one per rank). Per rank:
 *   1. lsa_score_chunks and lsa_topk_select on its own chunks with k_local = min(k, n_local);
 *   2. lsa_shard_candidates -> (score, global id) candidates, padded to k_pad with
 *      (-FLT_MAX, -1); the caller all-gathers them into [G][B][k_pad];
 *   3. lsa_shard_global_select -> the global keep set (the top-k of the candidates, ties to
 *      the lower global id) and this rank's share of it (local ids + count);
 *   4. lsa_sparse_decode_attn_counts over its share -> (out_g, lse_g); the caller all-gathers
 *      them into [G][B][H][Dh] and [G][B][H];
 *   5. lsa_merge_partials -> the step's output (log-sum-exp merge).
 * Scores must be greater than -FLT_MAX. */

/* Step 2. local_dims: this rank's shard (k / k_per_seq = its local candidate counts);
 * local_ids [sum k_local] from lsa_topk_select; global_offset host [B]: global id of the
 * rank's first chunk per sequence; cand_scores [B][k_pad] float32 and cand_ids [B][k_pad]
 * int32, out. */
LSA_API lsa_status lsa_shard_candidates(const lsa_dims *local_dims, const float *scores, const int32_t *local_ids,
                                        const int32_t *global_offset, int32_t k_pad, float *cand_scores,
                                        int32_t *cand_ids, void *stream);

/* Step 3. global_dims: B, N = G * k_pad, k / k_per_seq = the global k (no chunk_offsets);
 * global_offset, local_n host [B]: this rank's first global chunk id and chunk count per
 * sequence; all_scores [G][B][k_pad], all_ids [G][B][k_pad]: the gathered candidates;
 * seq_scores, seq_ids [B][G*k_pad]: caller scratch; global_ids [sum k] out (nullable): the
 * global keep set, ascending; local_ids [sum_b min(k_b, local_n_b)] out: this rank's kept
 * ids (local, ascending) then -1; local_count [B] out. ws: a workspace for global_dims. */
LSA_API lsa_status lsa_shard_global_select(const lsa_dims *global_dims, int32_t G, const int32_t *global_offset,
                                           const int32_t *local_n, const float *all_scores, const int32_t *all_ids,
                                           float *seq_scores, int32_t *seq_ids, int32_t *global_ids,
                                           int32_t *local_ids, int32_t *local_count, void *ws, size_t ws_bytes,
                                           void *stream);

/* Step 5. outs [G][B][H][Dh] float32 normalised outputs, lses [G][B][H] natural-log sums
 * (-inf for a rank that kept nothing); out [B][H][Dh], lse [B][H] (nullable):
 *   out = sum_g e^(lse_g - M) out_g / sum_g e^(lse_g - M),  lse = M + log sum_g e^(lse_g - M). */
LSA_API lsa_status lsa_merge_partials(int32_t G, int32_t B, int32_t H, const float *outs, const float *lses,
                                      float *out, float *lse, void *stream);

/* Synchronise `stream`, read the sticky device error word of `ws`, clear it, and
 * return LSA_OK or the first device error (NONFINITE, BAD_ID, TIMEOUT, in that order). */
LSA_API lsa_status lsa_get_device_status(void *ws, void *stream);

/* Measurement utility, not a step of the method: read `bytes` of device memory at `buf` with
 * 16-byte non-coherent loads and discard them (grid-stride, two 1024-thread CTAs per SM), so
 * that a caller can time a plain DRAM read stream, the ceiling of the read-only attention
 * stream, beside a copy benchmark. `buf` 16-byte aligned and `bytes` a multiple of 16, else
 * LSA_ERR_INVALID_ARG with nothing launched; the caller owns the buffer. Async on `stream`. */
LSA_API lsa_status lsa_read_stream(const void *buf, size_t bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* LSA_H_ */
