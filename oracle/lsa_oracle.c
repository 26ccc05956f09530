/*
 * lsa_oracle.c - plain float64 reference of the Lookahead Sparse Attention
 * (LSA) decode step of FlashMemory-DeepSeek-V4.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test suite, the package's smoke check and
 * the benchmark's CPU-baseline leg load this library. The product path (the
 * CUDA kernels behind include/lsa.h) never calls it, and the two share no code.
 *
 * Everything is computed in float64, one sequence at a time, with plain loops
 * in the order the definitions state; no blocking, fusion or reordering.
 * Inputs arrive already widened to double (bf16 and fp32 widen exactly).
 *
 * Sources (web pages about "FlashMemory-DeepSeek-V4: Lightning Index
 * Ultra-Long Context via Lookahead Sparse Attention", arXiv 2606.09079):
 *   - dimensionstp.github.io review, section 3-2 (2) "Neural Memory Indexer":
 *     the indexer scores every compressed-K chunk against the query side;
 *   - the arXiv abstract and the bayesiansapien wiki post "Key points": the
 *     indexer is a standard dual-encoder, i.e. relevance is the inner product
 *     of a query-side and a chunk-side embedding;
 *   - the review, section 3-2 (3) "Lookahead Sparse Attention", steps 4-7:
 *     score all chunks, keep a top-k mask, attend over the kept chunks only;
 *     the review, section 3-2 (2): layer scores are combined with a max.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

/*
 * Chunk relevance of one sequence (review section 3-2 (2); abstract: dual
 * encoder). q is [nq][e] (nq = 1 for one decode query, 64 for the lookahead
 * window), emb is [n][e]. For each chunk i:
 *     s[i] = max over j of  sum_d q[j][d] * emb[i][d].
 * With nq = 1 this is the plain inner product.
 */
void lsa_oracle_chunk_scores(int64_t n, int64_t nq, int64_t e,
                             const double *q, const double *emb, double *s)
{
    for (int64_t i = 0; i < n; ++i) {
        double best = -INFINITY;
        for (int64_t j = 0; j < nq; ++j) {
            double dot = 0.0;
            for (int64_t d = 0; d < e; ++d)
                dot += q[j * e + d] * emb[i * e + d];
            if (dot > best)
                best = dot;
        }
        s[i] = best;
    }
}

typedef struct {
    double s;
    int64_t i;
} scored_chunk;

/* (score descending, index ascending); -0.0 and +0.0 compare equal. */
static int by_score_then_index(const void *a, const void *b)
{
    const scored_chunk *x = (const scored_chunk *)a;
    const scored_chunk *y = (const scored_chunk *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    if (x->i < y->i) return -1;
    if (x->i > y->i) return 1;
    return 0;
}

static int by_index(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/*
 * Top-k keep mask (review section 3-2 (3), step 5). Order the n chunks by
 * score, highest first, ties to the lower chunk index; keep the first k;
 * write the kept indices to ids[k] in ascending order.
 * Returns 0, or -1 if a score is not finite or k is outside 1..n.
 */
int lsa_oracle_topk(int64_t n, const double *s, int64_t k, int32_t *ids)
{
    if (k < 1 || k > n)
        return -1;
    for (int64_t i = 0; i < n; ++i)
        if (!isfinite(s[i]))
            return -1;
    scored_chunk *order = (scored_chunk *)malloc((size_t)n * sizeof(scored_chunk));
    if (!order)
        return -1;
    for (int64_t i = 0; i < n; ++i) {
        order[i].s = s[i];
        order[i].i = i;
    }
    qsort(order, (size_t)n, sizeof(scored_chunk), by_score_then_index);
    for (int64_t j = 0; j < k; ++j)
        ids[j] = (int32_t)order[j].i;
    free(order);
    qsort(ids, (size_t)k, sizeof(int32_t), by_index);
    return 0;
}

/*
 * Exact softmax attention of one decode query over t tokens (review section
 * 3-2 (3), steps 6-7: attention over the kept chunks only). q is [h][dh],
 * K and V are [t][h][dh]. For every head:
 *     z_u   = scale * sum_d q[h][d] * K[u][h][d]
 *     p_u   = exp(z_u - m) / sum_w exp(z_w - m),   m = max_u z_u
 *     out   = sum_u p_u * V[u][h][.]
 *     lse   = m + log(sum_w exp(z_w - m))           (= log sum_u exp z_u)
 * z is scratch of length t supplied by the caller.
 */
void lsa_oracle_attention(int64_t t, int64_t h, int64_t dh, double scale,
                          const double *q, const double *K, const double *V,
                          double *out, double *lse, double *z)
{
    for (int64_t hh = 0; hh < h; ++hh) {
        double m = -INFINITY;
        for (int64_t u = 0; u < t; ++u) {
            double dot = 0.0;
            for (int64_t d = 0; d < dh; ++d)
                dot += q[hh * dh + d] * K[(u * h + hh) * dh + d];
            z[u] = scale * dot;
            if (z[u] > m)
                m = z[u];
        }
        double l = 0.0;
        for (int64_t u = 0; u < t; ++u)
            l += exp(z[u] - m);
        for (int64_t d = 0; d < dh; ++d)
            out[hh * dh + d] = 0.0;
        for (int64_t u = 0; u < t; ++u) {
            double p = exp(z[u] - m) / l;
            for (int64_t d = 0; d < dh; ++d)
                out[hh * dh + d] += p * V[(u * h + hh) * dh + d];
        }
        lse[hh] = m + log(l);
    }
}

/* Resident KV footprint of one sequence: kept tokens over context tokens. */
double lsa_oracle_footprint(int64_t k, int64_t chunk_len, int64_t context_len)
{
    return (double)(k * chunk_len) / (double)context_len;
}

/*
 * Neural Memory Indexer score on compressed-K chunks (review section 3-2 (2): per-head
 * queries q_h, chunk key k_i, fused head weights w_h, sigmoid of the ReLU-weighted sum;
 * section 3-2 (2): the per-layer scores are ensembled by max or mean). Inputs are the
 * dequantised values' factors: keys k [L][n][D] with per-chunk scales ks [L][n], queries
 * q [L][H][D] with per-head scales qs [L][H], weights w [L][H]. For every chunk i:
 *     v_l = sum_h w[l][h] * max(0, ks[l][i] * qs[l][h] * sum_d q[l][h][d] * k[l][i][d])
 *     s_l = 1 / (1 + exp(-v_l))
 *     s[i] = max_l s_l   (mean = 0)   or   (1/L) sum_l s_l   (mean = 1)
 */
void lsa_oracle_indexer_scores(int64_t n, int64_t L, int64_t H, int64_t D, int mean,
                               const double *k, const double *ks, const double *q,
                               const double *qs, const double *w, double *s)
{
    for (int64_t i = 0; i < n; ++i) {
        double comb = mean ? 0.0 : -INFINITY;
        for (int64_t l = 0; l < L; ++l) {
            double v = 0.0;
            for (int64_t h = 0; h < H; ++h) {
                double dot = 0.0;
                for (int64_t d = 0; d < D; ++d)
                    dot += q[(l * H + h) * D + d] * k[(l * n + i) * D + d];
                double a = ks[l * n + i] * qs[l * H + h] * dot;
                v += w[l * H + h] * (a > 0.0 ? a : 0.0);
            }
            double sl = 1.0 / (1.0 + exp(-v));
            if (mean)
                comb += sl;
            else if (sl > comb)
                comb = sl;
        }
        s[i] = mean ? comb / (double)L : comb;
    }
}
