// lsa_api.cu - the C ABI (include/lsa.h): host-side validation, launch plans,
// workspace layout and the kernel launches of the LSA decode step.
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "lsa_device.cuh"

namespace lsa {
cudaError_t launch_score(const lsa_dims& d, const SeqTable& tab, int max_n, const void* q_emb,
                         const void* chunk_emb, float* scores, uint32_t* err, int num_sms,
                         cudaStream_t stream, bool pdl);
bool score_uses_umma(const lsa_dims& d);
cudaError_t launch_topk(const lsa_dims& d, const SeqTable& tab, int max_n, const float* scores,
                        int32_t* ids, uint32_t* err, cudaStream_t stream, bool pdl);
cudaError_t launch_threshold(const lsa_dims& d, const SeqTable& tab, int max_n, const float* scores,
                             float tau, int k_min, int32_t* ids, int32_t* counts, uint32_t* err,
                             cudaStream_t stream, bool pdl);
cudaError_t launch_gather(const lsa_dims& d, const SeqTable& tab, const void* K, const void* V,
                          const int32_t* ids, void* K_res, void* V_res, uint32_t* err,
                          cudaStream_t stream);
cudaError_t attn_ctas_per_device(lsa_dtype kv, int num_sms, int* out);
bool small_step_eligible(const lsa_dims& d, int max_n, int64_t total_kept);
size_t small_step_part_bytes(const lsa_dims& d, int64_t total_kept);
cudaError_t launch_small_step(const lsa_dims& d, const SeqTable& tab, const void* q_emb, const void* chunk_emb,
                              const void* q, const void* K, const void* V, int32_t* ids, float* out, float* lse,
                              float* part, uint32_t* ws, cudaStream_t stream);
cudaError_t score_init_attrs();
cudaError_t topk_init_attrs();
cudaError_t refresh_init_attrs();
cudaError_t fp8_init_attrs();
struct ShardOffsets {
    int32_t global0[kMaxB];
};
cudaError_t launch_shard_candidates(const SeqTable& tab, int B, const ShardOffsets& offs, int k_pad,
                                    const float* scores, const int32_t* ids, float* cs, int32_t* ci,
                                    cudaStream_t st);
cudaError_t launch_shard_transpose(int G, int B, int k_pad, const float* in_s, const int32_t* in_i, float* out_s,
                                   int32_t* out_i, cudaStream_t st);
cudaError_t launch_shard_select(const int32_t* pos, const int32_t* cand_ids, const SeqTable& gtab,
                                const ShardOffsets& offs, const SeqTable& ltab, int B, int G, int k_pad,
                                int32_t* local_ids, int32_t* local_count, int32_t* global_ids, cudaStream_t st);
cudaError_t launch_merge_partials(const float* outs, const float* lses, int G, int B, int H, float* out, float* lse,
                                  cudaStream_t st);
cudaError_t launch_score_fp8(const lsa_dims& d, const SeqTable& tab, int max_n, int n_layers, int n_heads,
                             int mean, const uint8_t* ckv, const uint8_t* q8, const float* q_scale,
                             const float* head_w, float* scores, uint32_t* err, cudaStream_t stream,
                             bool pdl);
int refresh_max_chunks();
cudaError_t launch_refresh(const lsa_dims& d, const SeqTable& tab, int max_n, const int32_t* new_ids,
                           int32_t* slot_ids, const void* K, const void* V, void* K_res, void* V_res,
                           int32_t* copy_src, int32_t* copy_dst, int32_t* copy_count, int32_t* moved,
                           cudaStream_t stream);
cudaError_t la_init_attrs(int* ctas_per_sm);
int la_max_queries();
int64_t la_tiles(const lsa_dims& d, const SeqTable& tab);
int la_partition(const SeqTable& tab, int H, int max_ctas, int32_t* cta_start);
cudaError_t launch_attention_la(const lsa_dims& d, const SeqTable& tab, int max_ctas, const void* q, const void* K,
                                const void* V, int64_t kv_rows, const int32_t* ids, float* part_o, float* part_ml,
                                float* out, float* lse, uint32_t* err, cudaStream_t stream, bool pdl);
cudaError_t launch_attention(const lsa_dims& d, const SeqTable& tab, int ctas_per_device,
                             const void* q, const void* K, const void* V, const int32_t* ids,
                             float* part_o, float* part_ml, float* out, float* lse, uint32_t* err,
                             cudaStream_t stream, bool pdl, const int32_t* counts = nullptr);
}  // namespace lsa

using namespace lsa;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool ready;
    int sms;
    int attn_ctas[2];  // per kv dtype (LSA_F32, LSA_BF16)
    int la_ctas;       // CTAs of the lookahead-window attention
};

std::mutex g_dev_mu;
DeviceInfo g_dev[kMaxDevices];

// SM count and attention CTAs per device, computed once per device.
lsa_status device_info(DeviceInfo* out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LSA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_dev_mu);
    DeviceInfo& di = g_dev[dev];
    if (!di.ready) {
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return LSA_ERR_CUDA;
        di.sms = sms;
        // kernel attributes are per device: set them here, never inside a launch (graph capture)
        if (score_init_attrs() != cudaSuccess || topk_init_attrs() != cudaSuccess ||
            refresh_init_attrs() != cudaSuccess || fp8_init_attrs() != cudaSuccess)
            return LSA_ERR_CUDA;
        if (attn_ctas_per_device(LSA_F32, sms, &di.attn_ctas[LSA_F32]) != cudaSuccess) return LSA_ERR_CUDA;
        if (attn_ctas_per_device(LSA_BF16, sms, &di.attn_ctas[LSA_BF16]) != cudaSuccess) return LSA_ERR_CUDA;
        int la_occ = 0;
        if (la_init_attrs(&la_occ) != cudaSuccess || la_occ < 1) return LSA_ERR_CUDA;
        di.la_ctas = la_occ * sms;
        di.ready = true;
    }
    *out = di;
    return LSA_OK;
}

bool is_pow2(int64_t x) { return x > 0 && (x & (x - 1)) == 0; }
bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct Prepared {
    SeqTable tab;
    int max_n;
    int64_t total_chunks;
    int64_t total_kept;
};

// Validate the shape and build the per-sequence table.
lsa_status prepare(const lsa_dims* d, Prepared* p) {
    if (d == nullptr || p == nullptr) return LSA_ERR_INVALID_ARG;
    if (d->B < 1 || d->B > LSA_MAX_BATCH) return LSA_ERR_INVALID_ARG;
    if (d->Q < 1 || d->Q > 256 || d->E < 1) return LSA_ERR_INVALID_ARG;
    if (d->emb_dtype != LSA_F32 && d->emb_dtype != LSA_BF16) return LSA_ERR_INVALID_ARG;
    if (d->kv_dtype != LSA_F32 && d->kv_dtype != LSA_BF16) return LSA_ERR_INVALID_ARG;
    if (d->Dh != LSA_HEAD_DIM) return LSA_ERR_UNSUPPORTED;
    if (!is_pow2(d->H) || d->H > 128) return LSA_ERR_UNSUPPORTED;
    if (!is_pow2(d->chunk_len) || d->chunk_len < 8 || d->chunk_len > 1024) return LSA_ERR_UNSUPPORTED;
    const int es = d->emb_dtype == LSA_BF16 ? 2 : 4;
    const int64_t row_bytes = (int64_t)d->E * es;
    if (row_bytes % 16 != 0) return LSA_ERR_UNSUPPORTED;
    const int64_t pieces = row_bytes / 16;
    if (!((pieces <= 32 && is_pow2(pieces)) || pieces % 32 == 0)) return LSA_ERR_UNSUPPORTED;
    if (!score_uses_umma(*d) && (int64_t)d->Q * d->E * 4 > 200 * 1024) return LSA_ERR_UNSUPPORTED;

    SeqTable& t = p->tab;
    std::memset(&t, 0, sizeof(t));
    t.B = d->B;
    t.C = d->chunk_len;
    int64_t chunks = 0, kept = 0;
    int max_n = 0;
    for (int b = 0; b < d->B; ++b) {
        int64_t n;
        if (d->chunk_offsets) {
            if (b == 0 && d->chunk_offsets[0] != 0) return LSA_ERR_INVALID_ARG;
            n = d->chunk_offsets[b + 1] - d->chunk_offsets[b];
        } else {
            n = d->N;
        }
        const int64_t k = d->k_per_seq ? d->k_per_seq[b] : d->k;
        if (n < 1 || k < 1 || k > n) return LSA_ERR_INVALID_ARG;
        t.chunk_off[b] = (int32_t)chunks;
        t.kept_off[b] = (int32_t)kept;
        chunks += n;
        kept += k;
        if (chunks > (1ll << 30) || kept > (1ll << 30)) return LSA_ERR_UNSUPPORTED;
        if (n > max_n) max_n = (int)n;
    }
    t.chunk_off[d->B] = (int32_t)chunks;
    t.kept_off[d->B] = (int32_t)kept;
    p->max_n = max_n;
    p->total_chunks = chunks;
    p->total_kept = kept;
    return LSA_OK;
}

struct WsLayout {
    size_t scores, part_o, part_ml, ids, copy_src, copy_dst, copy_count, la_o, la_ml, small, total;
};

// The lookahead-window attention runs for bf16 K/V and windows of up to 64 queries.
bool la_shape(const lsa_dims* d) { return d->kv_dtype == LSA_BF16 && d->Q <= la_max_queries(); }

// Workspace: header (sticky error word; arrival counters of the one-launch step) | scores |
// split partials | refresh buffers | lookahead partials | one-launch step partials.
WsLayout ws_layout(const lsa_dims* d, const Prepared& p, const DeviceInfo& di) {
    WsLayout w;
    const int slots = di.attn_ctas[d->kv_dtype] + d->B;
    w.scores = kWsHeader;
    w.part_o = align256(w.scores + (size_t)p.total_chunks * 4);
    w.part_ml = align256(w.part_o + (size_t)slots * d->H * LSA_HEAD_DIM * 4);
    w.ids = align256(w.part_ml + (size_t)slots * d->H * 2 * 4);
    w.copy_src = align256(w.ids + (size_t)p.total_kept * 4);
    w.copy_dst = align256(w.copy_src + (size_t)p.total_kept * 4);
    w.copy_count = align256(w.copy_dst + (size_t)p.total_kept * 4);
    // lookahead partials: two slots per CTA (its first and last (sequence, head) run)
    const size_t la_slots = la_shape(d) ? (size_t)2 * di.la_ctas : 0;
    w.la_o = align256(w.copy_count + (size_t)d->B * 4);
    w.la_ml = align256(w.la_o + la_slots * d->Q * LSA_HEAD_DIM * 4);
    // partials of the one-launch step (small problems only)
    w.small = align256(w.la_ml + la_slots * d->Q * 2 * 4);
    const size_t small_bytes = small_step_eligible(*d, p.max_n, p.total_kept) ? small_step_part_bytes(*d, p.total_kept) : 0;
    w.total = align256(w.small + small_bytes);
    return w;
}

// Validation shared by every call that takes a workspace.
lsa_status prepare_ws(const lsa_dims* d, void* ws, size_t ws_bytes, Prepared* p, DeviceInfo* di,
                      WsLayout* w) {
    lsa_status s = prepare(d, p);
    if (s != LSA_OK) return s;
    if (!aligned16(ws)) return LSA_ERR_INVALID_ARG;
    s = device_info(di);
    if (s != LSA_OK) return s;
    *w = ws_layout(d, *p, *di);
    if (ws_bytes < w->total) return LSA_ERR_WORKSPACE;
    return LSA_OK;
}

inline uint8_t* at(void* ws, size_t off) { return static_cast<uint8_t*>(ws) + off; }
inline lsa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? LSA_OK : LSA_ERR_CUDA; }

}  // namespace

extern "C" {

int lsa_abi_version(void) { return LSA_ABI_VERSION; }

const char* lsa_status_string(lsa_status s) {
    switch (s) {
        case LSA_OK: return "LSA_OK";
        case LSA_ERR_INVALID_ARG: return "LSA_ERR_INVALID_ARG: invalid argument";
        case LSA_ERR_WORKSPACE: return "LSA_ERR_WORKSPACE: workspace too small";
        case LSA_ERR_CUDA: return "LSA_ERR_CUDA: CUDA runtime error";
        case LSA_ERR_NONFINITE: return "LSA_ERR_NONFINITE: non-finite chunk score";
        case LSA_ERR_TIMEOUT: return "LSA_ERR_TIMEOUT: a bounded device wait gave up";
        case LSA_ERR_UNSUPPORTED: return "LSA_ERR_UNSUPPORTED: shape not implemented";
        case LSA_ERR_BAD_ID: return "LSA_ERR_BAD_ID: kept chunk id out of range";
    }
    return "LSA_ERR_?: unknown status";
}

lsa_status lsa_workspace_size(const lsa_dims* dims, size_t* bytes) {
    if (bytes == nullptr) return LSA_ERR_INVALID_ARG;
    Prepared p;
    lsa_status s = prepare(dims, &p);
    if (s != LSA_OK) return s;
    DeviceInfo di;
    s = device_info(&di);
    if (s != LSA_OK) return s;
    *bytes = ws_layout(dims, p, di).total;
    return LSA_OK;
}

lsa_status lsa_workspace_init(void* ws, size_t ws_bytes, void* stream) {
    if (!aligned16(ws) || ws_bytes < kWsHeader) return LSA_ERR_INVALID_ARG;
    return cuda_status(cudaMemsetAsync(ws, 0, kWsHeader, static_cast<cudaStream_t>(stream)));
}

lsa_status lsa_score_chunks(const lsa_dims* dims, const void* q_emb, const void* chunk_emb,
                            float* scores, void* ws, size_t ws_bytes, void* stream) {
    Prepared p;
    DeviceInfo di;
    WsLayout w;
    lsa_status s = prepare_ws(dims, ws, ws_bytes, &p, &di, &w);
    if (s != LSA_OK) return s;
    if (!aligned16(q_emb) || !aligned16(chunk_emb) || !aligned16(scores)) return LSA_ERR_INVALID_ARG;
    return cuda_status(launch_score(*dims, p.tab, p.max_n, q_emb, chunk_emb, scores,
                                    reinterpret_cast<uint32_t*>(ws), di.sms,
                                    static_cast<cudaStream_t>(stream), false));
}

lsa_status lsa_topk_select(const lsa_dims* dims, const float* scores, int32_t* chunk_ids, void* ws,
                           size_t ws_bytes, void* stream) {
    Prepared p;
    DeviceInfo di;
    WsLayout w;
    lsa_status s = prepare_ws(dims, ws, ws_bytes, &p, &di, &w);
    if (s != LSA_OK) return s;
    if (!aligned16(scores) || !aligned16(chunk_ids)) return LSA_ERR_INVALID_ARG;
    return cuda_status(launch_topk(*dims, p.tab, p.max_n, scores, chunk_ids,
                                   reinterpret_cast<uint32_t*>(ws), static_cast<cudaStream_t>(stream),
                                   false));
}

lsa_status lsa_gather_kv(const lsa_dims* dims, const void* K, const void* V, const int32_t* chunk_ids,
                         void* K_res, void* V_res, void* ws, size_t ws_bytes, void* stream) {
    Prepared p;
    DeviceInfo di;
    WsLayout w;
    lsa_status s = prepare_ws(dims, ws, ws_bytes, &p, &di, &w);
    if (s != LSA_OK) return s;
    if (!aligned16(K) || !aligned16(V) || !aligned16(chunk_ids) || !aligned16(K_res) || !aligned16(V_res))
        return LSA_ERR_INVALID_ARG;
    return cuda_status(launch_gather(*dims, p.tab, K, V, chunk_ids, K_res, V_res,
                                     reinterpret_cast<uint32_t*>(ws), static_cast<cudaStream_t>(stream)));
}

lsa_status lsa_sparse_decode_attn(const lsa_dims* dims, const void* q, const void* K, const void* V,
                                  const int32_t* chunk_ids, float* out, float* lse, void* ws,
                                  size_t ws_bytes, void* stream) {
    Prepared p;
    DeviceInfo di;
    WsLayout w;
    lsa_status s = prepare_ws(dims, ws, ws_bytes, &p, &di, &w);
    if (s != LSA_OK) return s;
    if (!aligned16(q) || !aligned16(K) || !aligned16(V) || !aligned16(out)) return LSA_ERR_INVALID_ARG;
    if (chunk_ids != nullptr && !aligned16(chunk_ids)) return LSA_ERR_INVALID_ARG;
    if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) return LSA_ERR_INVALID_ARG;
    return cuda_status(launch_attention(*dims, p.tab, di.attn_ctas[dims->kv_dtype], q, K, V, chunk_ids,
                                        reinterpret_cast<float*>(at(ws, w.part_o)),
                                        reinterpret_cast<float*>(at(ws, w.part_ml)), out, lse,
                                        reinterpret_cast<uint32_t*>(ws),
                                        static_cast<cudaStream_t>(stream), false));
}

lsa_status lsa_decode_step(const lsa_dims* dims, const void* q_emb, const void* chunk_emb,
                           const void* q, const void* K, const void* V, int32_t* chunk_ids_out,
                           float* out, float* lse, void* ws, size_t ws_bytes, void* stream) {
    Prepared p;
    DeviceInfo di;
    WsLayout w;
    lsa_status s = prepare_ws(dims, ws, ws_bytes, &p, &di, &w);
    if (s != LSA_OK) return s;
    if (!aligned16(q_emb) || !aligned16(chunk_emb) || !aligned16(q) || !aligned16(K) ||
        !aligned16(V) || !aligned16(chunk_ids_out) || !aligned16(out))
        return LSA_ERR_INVALID_ARG;
    if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) return LSA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t* err = reinterpret_cast<uint32_t*>(ws);
    if (small_step_eligible(*dims, p.max_n, p.total_kept)) {
        // a few short sequences: the whole step in one launch
        return cuda_status(launch_small_step(*dims, p.tab, q_emb, chunk_emb, q, K, V, chunk_ids_out, out, lse,
                                             reinterpret_cast<float*>(at(ws, w.small)), err, st));
    }
    float* scores = reinterpret_cast<float*>(at(ws, w.scores));
    cudaError_t e = launch_score(*dims, p.tab, p.max_n, q_emb, chunk_emb, scores, err, di.sms, st, false);
    if (e != cudaSuccess) return LSA_ERR_CUDA;
    e = launch_topk(*dims, p.tab, p.max_n, scores, chunk_ids_out, err, st, true);
    if (e != cudaSuccess) return LSA_ERR_CUDA;
    e = launch_attention(*dims, p.tab, di.attn_ctas[dims->kv_dtype], q, K, V, chunk_ids_out,
                         reinterpret_cast<float*>(at(ws, w.part_o)),
                         reinterpret_cast<float*>(at(ws, w.part_ml)), out, lse, err, st, true);
    return cuda_status(e);
}

}  // extern "C"

namespace {

// Shape checks of the lookahead-window attention; rows of the K/V tensors it reads.
lsa_status la_check(const lsa_dims* d, const Prepared& p, bool indexed, int64_t* kv_rows) {
    if (d->kv_dtype != LSA_BF16) return LSA_ERR_UNSUPPORTED;
    if (d->Q > la_max_queries()) return LSA_ERR_UNSUPPORTED;
    const int64_t rows = (indexed ? p.total_chunks : p.total_kept) * (int64_t)d->chunk_len;
    if (rows >= (1ll << 31) || la_tiles(*d, p.tab) >= (1ll << 31)) return LSA_ERR_UNSUPPORTED;
    *kv_rows = rows;
    return LSA_OK;
}

}  // namespace

extern "C" {

lsa_status lsa_sparse_decode_attn_lookahead(const lsa_dims* dims, const void* q, const void* K, const void* V,
                                            const int32_t* chunk_ids, float* out, float* lse, void* ws,
                                            size_t ws_bytes, void* stream) {
    Prepared p;
    DeviceInfo di;
    WsLayout w;
    lsa_status s = prepare_ws(dims, ws, ws_bytes, &p, &di, &w);
    if (s != LSA_OK) return s;
    int64_t kv_rows = 0;
    s = la_check(dims, p, chunk_ids != nullptr, &kv_rows);
    if (s != LSA_OK) return s;
    if (!aligned16(q) || !aligned16(K) || !aligned16(V) || !aligned16(out)) return LSA_ERR_INVALID_ARG;
    if (chunk_ids != nullptr && !aligned16(chunk_ids)) return LSA_ERR_INVALID_ARG;
    if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) return LSA_ERR_INVALID_ARG;
    // programmatic dependent launch: every global read of the kernel follows its grid-dependency
    // wait, so only its prologue (TMEM, barriers) overlaps the previous kernel in the stream
    return cuda_status(launch_attention_la(*dims, p.tab, di.la_ctas, q, K, V, kv_rows, chunk_ids,
                                           reinterpret_cast<float*>(at(ws, w.la_o)),
                                           reinterpret_cast<float*>(at(ws, w.la_ml)), out, lse,
                                           reinterpret_cast<uint32_t*>(ws), static_cast<cudaStream_t>(stream),
                                           true));
}

lsa_status lsa_lookahead_partition(const lsa_dims* dims, int32_t max_ctas, int32_t* cta_start, int32_t* n_ctas) {
    if (cta_start == nullptr || n_ctas == nullptr || max_ctas < 1) return LSA_ERR_INVALID_ARG;
    Prepared p;
    lsa_status s = prepare(dims, &p);
    if (s != LSA_OK) return s;
    int64_t kv_rows = 0;
    s = la_check(dims, p, false, &kv_rows);
    if (s != LSA_OK) return s;
    *n_ctas = la_partition(p.tab, dims->H, max_ctas, cta_start);
    return LSA_OK;
}

lsa_status lsa_decode_step_lookahead(const lsa_dims* dims, const void* q_emb, const void* chunk_emb, const void* q,
                                     const void* K, const void* V, int32_t* chunk_ids_out, float* out, float* lse,
                                     void* ws, size_t ws_bytes, void* stream) {
    Prepared p;
    DeviceInfo di;
    WsLayout w;
    lsa_status s = prepare_ws(dims, ws, ws_bytes, &p, &di, &w);
    if (s != LSA_OK) return s;
    int64_t kv_rows = 0;
    s = la_check(dims, p, true, &kv_rows);
    if (s != LSA_OK) return s;
    if (!aligned16(q_emb) || !aligned16(chunk_emb) || !aligned16(q) || !aligned16(K) || !aligned16(V) ||
        !aligned16(chunk_ids_out) || !aligned16(out))
        return LSA_ERR_INVALID_ARG;
    if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) return LSA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t* err = reinterpret_cast<uint32_t*>(ws);
    float* scores = reinterpret_cast<float*>(at(ws, w.scores));
    cudaError_t e = launch_score(*dims, p.tab, p.max_n, q_emb, chunk_emb, scores, err, di.sms, st, false);
    if (e != cudaSuccess) return LSA_ERR_CUDA;
    e = launch_topk(*dims, p.tab, p.max_n, scores, chunk_ids_out, err, st, true);
    if (e != cudaSuccess) return LSA_ERR_CUDA;
    e = launch_attention_la(*dims, p.tab, di.la_ctas, q, K, V, kv_rows, chunk_ids_out,
                            reinterpret_cast<float*>(at(ws, w.la_o)), reinterpret_cast<float*>(at(ws, w.la_ml)),
                            out, lse, err, st, true);
    return cuda_status(e);
}

lsa_status lsa_threshold_select(const lsa_dims* dims, const float* scores, float tau, int32_t k_min,
                                int32_t* chunk_ids, int32_t* kept_count, void* ws, size_t ws_bytes,
                                void* stream) {
    Prepared p;
    DeviceInfo di;
    WsLayout w;
    lsa_status s = prepare_ws(dims, ws, ws_bytes, &p, &di, &w);
    if (s != LSA_OK) return s;
    if (!aligned16(scores) || !aligned16(chunk_ids) || !aligned16(kept_count)) return LSA_ERR_INVALID_ARG;
    if (k_min < 1 || !std::isfinite(tau)) return LSA_ERR_INVALID_ARG;
    return cuda_status(launch_threshold(*dims, p.tab, p.max_n, scores, tau, k_min, chunk_ids, kept_count,
                                        reinterpret_cast<uint32_t*>(ws), static_cast<cudaStream_t>(stream),
                                        false));
}

lsa_status lsa_decode_step_threshold(const lsa_dims* dims, const void* q_emb, const void* chunk_emb,
                                     const void* q, const void* K, const void* V, float tau, int32_t k_min,
                                     int32_t* chunk_ids_out, int32_t* kept_count_out, float* out, float* lse,
                                     void* ws, size_t ws_bytes, void* stream) {
    Prepared p;
    DeviceInfo di;
    WsLayout w;
    lsa_status s = prepare_ws(dims, ws, ws_bytes, &p, &di, &w);
    if (s != LSA_OK) return s;
    if (!aligned16(q_emb) || !aligned16(chunk_emb) || !aligned16(q) || !aligned16(K) || !aligned16(V) ||
        !aligned16(chunk_ids_out) || !aligned16(kept_count_out) || !aligned16(out))
        return LSA_ERR_INVALID_ARG;
    if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) return LSA_ERR_INVALID_ARG;
    if (k_min < 1 || !std::isfinite(tau)) return LSA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t* err = reinterpret_cast<uint32_t*>(ws);
    float* scores = reinterpret_cast<float*>(at(ws, w.scores));
    cudaError_t e = launch_score(*dims, p.tab, p.max_n, q_emb, chunk_emb, scores, err, di.sms, st, false);
    if (e == cudaSuccess)
        e = launch_threshold(*dims, p.tab, p.max_n, scores, tau, k_min, chunk_ids_out, kept_count_out, err, st, true);
    if (e == cudaSuccess)
        e = launch_attention(*dims, p.tab, di.attn_ctas[dims->kv_dtype], q, K, V, chunk_ids_out,
                             reinterpret_cast<float*>(at(ws, w.part_o)),
                             reinterpret_cast<float*>(at(ws, w.part_ml)), out, lse, err, st, true, kept_count_out);
    return cuda_status(e);
}

namespace {
lsa_status check_fp8_args(const lsa_dims* d, int32_t n_layers, int32_t n_heads, lsa_ensemble ens,
                          const void* ckv, const void* q8, const float* q_scale, const float* head_w) {
    if (d->E != LSA_INDEX_DIM) return LSA_ERR_INVALID_ARG;
    if (n_layers < 1 || n_layers > 16) return LSA_ERR_INVALID_ARG;
    if (n_heads < 16 || n_heads > 256 || n_heads % 16 != 0) return LSA_ERR_UNSUPPORTED;
    if (ens != LSA_ENSEMBLE_MAX && ens != LSA_ENSEMBLE_MEAN) return LSA_ERR_INVALID_ARG;
    if (!aligned16(ckv) || !aligned16(q8)) return LSA_ERR_INVALID_ARG;
    if (q_scale == nullptr || head_w == nullptr || (reinterpret_cast<uintptr_t>(q_scale) & 3u) ||
        (reinterpret_cast<uintptr_t>(head_w) & 3u))
        return LSA_ERR_INVALID_ARG;
    return LSA_OK;
}
}  // namespace

lsa_status lsa_indexer_score_fp8(const lsa_dims* dims, int32_t n_layers, int32_t n_heads, lsa_ensemble ensemble,
                                 const void* compressed_k, const void* q_fp8, const float* q_scale,
                                 const float* head_w, float* scores, void* ws, size_t ws_bytes, void* stream) {
    Prepared p;
    DeviceInfo di;
    WsLayout w;
    lsa_status s = prepare_ws(dims, ws, ws_bytes, &p, &di, &w);
    if (s != LSA_OK) return s;
    s = check_fp8_args(dims, n_layers, n_heads, ensemble, compressed_k, q_fp8, q_scale, head_w);
    if (s != LSA_OK) return s;
    if (!aligned16(scores)) return LSA_ERR_INVALID_ARG;
    return cuda_status(launch_score_fp8(*dims, p.tab, p.max_n, n_layers, n_heads, ensemble == LSA_ENSEMBLE_MEAN,
                                        static_cast<const uint8_t*>(compressed_k), static_cast<const uint8_t*>(q_fp8),
                                        q_scale, head_w, scores, reinterpret_cast<uint32_t*>(ws),
                                        static_cast<cudaStream_t>(stream), false));
}

lsa_status lsa_decode_step_fp8(const lsa_dims* dims, int32_t n_layers, int32_t n_heads, lsa_ensemble ensemble,
                               const void* compressed_k, const void* q_fp8, const float* q_scale,
                               const float* head_w, const void* q, const void* K, const void* V,
                               int32_t* chunk_ids_out, float* out, float* lse, void* ws, size_t ws_bytes,
                               void* stream) {
    Prepared p;
    DeviceInfo di;
    WsLayout w;
    lsa_status s = prepare_ws(dims, ws, ws_bytes, &p, &di, &w);
    if (s != LSA_OK) return s;
    s = check_fp8_args(dims, n_layers, n_heads, ensemble, compressed_k, q_fp8, q_scale, head_w);
    if (s != LSA_OK) return s;
    if (!aligned16(q) || !aligned16(K) || !aligned16(V) || !aligned16(chunk_ids_out) || !aligned16(out))
        return LSA_ERR_INVALID_ARG;
    if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) return LSA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t* err = reinterpret_cast<uint32_t*>(ws);
    float* scores = reinterpret_cast<float*>(at(ws, w.scores));
    cudaError_t e = launch_score_fp8(*dims, p.tab, p.max_n, n_layers, n_heads, ensemble == LSA_ENSEMBLE_MEAN,
                                     static_cast<const uint8_t*>(compressed_k), static_cast<const uint8_t*>(q_fp8),
                                     q_scale, head_w, scores, err, st, false);
    if (e == cudaSuccess) e = launch_topk(*dims, p.tab, p.max_n, scores, chunk_ids_out, err, st, true);
    if (e == cudaSuccess)
        e = launch_attention(*dims, p.tab, di.attn_ctas[dims->kv_dtype], q, K, V, chunk_ids_out,
                             reinterpret_cast<float*>(at(ws, w.part_o)),
                             reinterpret_cast<float*>(at(ws, w.part_ml)), out, lse, err, st, true);
    return cuda_status(e);
}

lsa_status lsa_sparse_decode_attn_counts(const lsa_dims* dims, const void* q, const void* K, const void* V,
                                         const int32_t* chunk_ids, const int32_t* kept_count, float* out,
                                         float* lse, void* ws, size_t ws_bytes, void* stream) {
    Prepared p;
    DeviceInfo di;
    WsLayout w;
    lsa_status s = prepare_ws(dims, ws, ws_bytes, &p, &di, &w);
    if (s != LSA_OK) return s;
    if (!aligned16(q) || !aligned16(K) || !aligned16(V) || !aligned16(chunk_ids) || !aligned16(kept_count) ||
        !aligned16(out))
        return LSA_ERR_INVALID_ARG;
    if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) return LSA_ERR_INVALID_ARG;
    return cuda_status(launch_attention(*dims, p.tab, di.attn_ctas[dims->kv_dtype], q, K, V, chunk_ids,
                                        reinterpret_cast<float*>(at(ws, w.part_o)),
                                        reinterpret_cast<float*>(at(ws, w.part_ml)), out, lse,
                                        reinterpret_cast<uint32_t*>(ws), static_cast<cudaStream_t>(stream), false,
                                        kept_count));
}

lsa_status lsa_shard_candidates(const lsa_dims* local_dims, const float* scores, const int32_t* local_ids,
                                const int32_t* global_offset, int32_t k_pad, float* cand_scores,
                                int32_t* cand_ids, void* stream) {
    Prepared p;
    lsa_status s = prepare(local_dims, &p);
    if (s != LSA_OK) return s;
    if (global_offset == nullptr || !aligned16(scores) || !aligned16(local_ids) || !aligned16(cand_scores) ||
        !aligned16(cand_ids))
        return LSA_ERR_INVALID_ARG;
    ShardOffsets offs;
    std::memset(&offs, 0, sizeof(offs));
    for (int b = 0; b < local_dims->B; ++b) {
        const int kb = p.tab.kept_off[b + 1] - p.tab.kept_off[b];
        if (global_offset[b] < 0 || kb > k_pad) return LSA_ERR_INVALID_ARG;
        offs.global0[b] = global_offset[b];
    }
    if (k_pad < 1) return LSA_ERR_INVALID_ARG;
    return cuda_status(launch_shard_candidates(p.tab, local_dims->B, offs, k_pad, scores, local_ids, cand_scores,
                                               cand_ids, static_cast<cudaStream_t>(stream)));
}

lsa_status lsa_shard_global_select(const lsa_dims* global_dims, int32_t G, const int32_t* global_offset,
                                   const int32_t* local_n, const float* all_scores, const int32_t* all_ids,
                                   float* seq_scores, int32_t* seq_ids, int32_t* global_ids, int32_t* local_ids,
                                   int32_t* local_count, void* ws, size_t ws_bytes, void* stream) {
    Prepared gp;
    DeviceInfo di;
    WsLayout w;
    lsa_status s = prepare_ws(global_dims, ws, ws_bytes, &gp, &di, &w);
    if (s != LSA_OK) return s;
    if (global_dims->chunk_offsets != nullptr || G < 1 || global_dims->N % G != 0) return LSA_ERR_INVALID_ARG;
    if (global_offset == nullptr || local_n == nullptr || !aligned16(all_scores) || !aligned16(all_ids) ||
        !aligned16(seq_scores) || !aligned16(seq_ids) || !aligned16(local_ids) || !aligned16(local_count) ||
        (global_ids != nullptr && !aligned16(global_ids)))
        return LSA_ERR_INVALID_ARG;
    const int k_pad = global_dims->N / G;
    const int B = global_dims->B;
    // this rank's local table: its chunk counts, and one slot per globally kept chunk as capacity
    SeqTable ltab;
    std::memset(&ltab, 0, sizeof(ltab));
    ltab.B = B;
    ltab.C = global_dims->chunk_len;
    ShardOffsets offs;
    std::memset(&offs, 0, sizeof(offs));
    int64_t chunks = 0, cap = 0;
    for (int b = 0; b < B; ++b) {
        if (local_n[b] < 1 || global_offset[b] < 0) return LSA_ERR_INVALID_ARG;
        const int kb = gp.tab.kept_off[b + 1] - gp.tab.kept_off[b];
        ltab.chunk_off[b] = (int32_t)chunks;
        ltab.kept_off[b] = (int32_t)cap;
        chunks += local_n[b];
        cap += kb < local_n[b] ? kb : local_n[b];  // a rank keeps at most min(k, its chunks)
        offs.global0[b] = global_offset[b];
    }
    ltab.chunk_off[B] = (int32_t)chunks;
    ltab.kept_off[B] = (int32_t)cap;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t* pos = reinterpret_cast<int32_t*>(at(ws, w.ids));
    cudaError_t e = launch_shard_transpose(G, B, k_pad, all_scores, all_ids, seq_scores, seq_ids, st);
    if (e == cudaSuccess)
        e = launch_topk(*global_dims, gp.tab, gp.max_n, seq_scores, pos, reinterpret_cast<uint32_t*>(ws), st, false);
    if (e == cudaSuccess)
        e = launch_shard_select(pos, seq_ids, gp.tab, offs, ltab, B, G, k_pad, local_ids, local_count, global_ids, st);
    return cuda_status(e);
}

lsa_status lsa_merge_partials(int32_t G, int32_t B, int32_t H, const float* outs, const float* lses, float* out,
                              float* lse, void* stream) {
    if (G < 1 || B < 1 || H < 1 || H > 65535 || B > 65535) return LSA_ERR_INVALID_ARG;
    if (!aligned16(outs) || !aligned16(lses) || !aligned16(out)) return LSA_ERR_INVALID_ARG;
    if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) return LSA_ERR_INVALID_ARG;
    return cuda_status(launch_merge_partials(outs, lses, G, B, H, out, lse, static_cast<cudaStream_t>(stream)));
}

lsa_status lsa_refresh_resident(const lsa_dims* dims, const void* q_emb, const void* chunk_emb,
                                const void* K, const void* V, int32_t* slot_ids, void* K_res,
                                void* V_res, int32_t* moved, void* ws, size_t ws_bytes, void* stream) {
    Prepared p;
    DeviceInfo di;
    WsLayout w;
    lsa_status s = prepare_ws(dims, ws, ws_bytes, &p, &di, &w);
    if (s != LSA_OK) return s;
    if (!aligned16(q_emb) || !aligned16(chunk_emb) || !aligned16(K) || !aligned16(V) ||
        !aligned16(slot_ids) || !aligned16(K_res) || !aligned16(V_res))
        return LSA_ERR_INVALID_ARG;
    if (moved != nullptr && (reinterpret_cast<uintptr_t>(moved) & 3u)) return LSA_ERR_INVALID_ARG;
    if (p.max_n > refresh_max_chunks()) return LSA_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t* err = reinterpret_cast<uint32_t*>(ws);
    float* scores = reinterpret_cast<float*>(at(ws, w.scores));
    int32_t* ids = reinterpret_cast<int32_t*>(at(ws, w.ids));
    cudaError_t e = launch_score(*dims, p.tab, p.max_n, q_emb, chunk_emb, scores, err, di.sms, st, false);
    if (e == cudaSuccess) e = launch_topk(*dims, p.tab, p.max_n, scores, ids, err, st, true);
    if (e == cudaSuccess)
        e = launch_refresh(*dims, p.tab, p.max_n, ids, slot_ids, K, V, K_res, V_res,
                           reinterpret_cast<int32_t*>(at(ws, w.copy_src)),
                           reinterpret_cast<int32_t*>(at(ws, w.copy_dst)),
                           reinterpret_cast<int32_t*>(at(ws, w.copy_count)), moved, st);
    return cuda_status(e);
}

lsa_status lsa_get_device_status(void* ws, void* stream) {
    if (!aligned16(ws)) return LSA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return LSA_ERR_CUDA;
    uint32_t word = 0;
    if (cudaMemcpy(&word, ws, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return LSA_ERR_CUDA;
    if (word != 0 && cudaMemset(ws, 0, sizeof(word)) != cudaSuccess) return LSA_ERR_CUDA;
    if (word & kErrNonFinite) return LSA_ERR_NONFINITE;
    if (word & kErrBadId) return LSA_ERR_BAD_ID;
    if (word & kErrTimeout) return LSA_ERR_TIMEOUT;
    return LSA_OK;
}

}  // extern "C"
