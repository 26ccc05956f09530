// noalloc.cu - lsa_sparse_decode_attn_noalloc: the sparse decode attention call
// for callers that cannot allocate device memory.
//
// Who needs it: lsa_sparse_decode_attn writes its split-K partial results to a
// caller-provided workspace, which the caller must obtain with cudaMalloc (or a
// caching allocator on top of it). Some callers cannot do that: an inference
// engine that has already reserved almost all device memory for its own pool, a
// plugin running inside another framework that must not allocate behind that
// framework's allocator, or a latency-critical loop where cudaMalloc's implicit
// device-wide synchronisation is not acceptable. This entry point keeps its
// scratch in a fixed array compiled into the library instead.
//
// The scratch: `g_noalloc_scratch`, kNoallocScratchBytes (4 MiB) of device memory
// per GPU that loads the library, held until the process exits. It is shared by
// every call on that GPU and keeps the last call's contents; the part that must
// start at zero (the device error word) is cleared by each call. Calls whose
// kernels overlap on the GPU (different streams without ordering between them)
// race on the array: order them on one stream.
//
// Host code never dereferences the array's name: on the host it is only a stand-in
// for the symbol. The device address comes from cudaGetSymbolAddress, taken once
// per device (with that device current) on the first call made on the device.
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

#include "lsa_device.cuh"

namespace lsa {
cudaError_t attn_ctas_per_device(lsa_dtype kv, int num_sms, int* out);
cudaError_t launch_attention(const lsa_dims& d, const SeqTable& tab, int ctas_per_device,
                             const void* q, const void* K, const void* V, const int32_t* ids,
                             float* part_o, float* part_ml, float* out, float* lse, uint32_t* err,
                             cudaStream_t stream, bool pdl, const int32_t* counts = nullptr);
}  // namespace lsa

using namespace lsa;

namespace {

constexpr size_t kNoallocScratchBytes = (size_t)4 << 20;  // LSA_NOALLOC_SCRATCH_BYTES
static_assert(kNoallocScratchBytes == LSA_NOALLOC_SCRATCH_BYTES, "header and library disagree");

// Layout: [0, 256) error word | split partials (o) | split partials (m, l).
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDev = 64;

struct NoallocDevice {
    bool ready;
    uint8_t* scratch;  // device address of g_noalloc_scratch on this device
    int sms;
    int attn_ctas[2];
};

std::mutex g_mu;
NoallocDevice g_devs[kMaxDev];

// One-time set-up per device, with that device current.
lsa_status noalloc_device(NoallocDevice* out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return LSA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    NoallocDevice& d = g_devs[dev];
    if (!d.ready) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return LSA_ERR_CUDA;
        d.scratch = static_cast<uint8_t*>(p);
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return LSA_ERR_CUDA;
        if (attn_ctas_per_device(LSA_F32, d.sms, &d.attn_ctas[LSA_F32]) != cudaSuccess) return LSA_ERR_CUDA;
        if (attn_ctas_per_device(LSA_BF16, d.sms, &d.attn_ctas[LSA_BF16]) != cudaSuccess) return LSA_ERR_CUDA;
        d.ready = true;
    }
    *out = d;
    return LSA_OK;
}

bool pow2(int64_t x) { return x > 0 && (x & (x - 1)) == 0; }
bool al16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

extern "C" LSA_API lsa_status lsa_sparse_decode_attn_noalloc(const lsa_dims* d, const void* q,
                                                             const void* K, const void* V,
                                                             const int32_t* chunk_ids, float* out,
                                                             float* lse, void* stream) {
    // ---- the same shape checks as the workspace entry point
    if (d == nullptr) return LSA_ERR_INVALID_ARG;
    if (d->B < 1 || d->B > LSA_MAX_BATCH || d->Q < 1 || d->Q > 256 || d->E < 1) return LSA_ERR_INVALID_ARG;
    if (d->emb_dtype != LSA_F32 && d->emb_dtype != LSA_BF16) return LSA_ERR_INVALID_ARG;
    if (d->kv_dtype != LSA_F32 && d->kv_dtype != LSA_BF16) return LSA_ERR_INVALID_ARG;
    if (d->Dh != LSA_HEAD_DIM || !pow2(d->H) || d->H > 128) return LSA_ERR_UNSUPPORTED;
    if (!pow2(d->chunk_len) || d->chunk_len < 8 || d->chunk_len > 1024) return LSA_ERR_UNSUPPORTED;
    if (!al16(q) || !al16(K) || !al16(V) || !al16(out)) return LSA_ERR_INVALID_ARG;
    if (chunk_ids != nullptr && !al16(chunk_ids)) return LSA_ERR_INVALID_ARG;
    if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) return LSA_ERR_INVALID_ARG;
    SeqTable tab;
    std::memset(&tab, 0, sizeof(tab));
    tab.B = d->B;
    tab.C = d->chunk_len;
    int64_t chunks = 0, kept = 0;
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
        tab.chunk_off[b] = (int32_t)chunks;
        tab.kept_off[b] = (int32_t)kept;
        chunks += n;
        kept += k;
        if (chunks > (1ll << 30) || kept > (1ll << 30)) return LSA_ERR_UNSUPPORTED;
    }
    tab.chunk_off[d->B] = (int32_t)chunks;
    tab.kept_off[d->B] = (int32_t)kept;

    NoallocDevice dev;
    lsa_status s = noalloc_device(&dev);
    if (s != LSA_OK) return s;

    // ---- the partials must fit in the fixed scratch: reject larger shapes before launching
    const int ctas = dev.attn_ctas[d->kv_dtype];
    const size_t slots = (size_t)ctas + d->B;
    const size_t off_o = kWsHeader;
    const size_t off_ml = up256(off_o + slots * d->H * LSA_HEAD_DIM * 4);
    const size_t need = up256(off_ml + slots * d->H * 2 * 4);
    if (need > kNoallocScratchBytes) return LSA_ERR_WORKSPACE;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t* err = reinterpret_cast<uint32_t*>(dev.scratch);
    if (cudaMemsetAsync(err, 0, sizeof(uint32_t), st) != cudaSuccess) return LSA_ERR_CUDA;
    const cudaError_t e = launch_attention(*d, tab, ctas, q, K, V, chunk_ids,
                                           reinterpret_cast<float*>(dev.scratch + off_o),
                                           reinterpret_cast<float*>(dev.scratch + off_ml), out, lse, err,
                                           st, false);
    return e == cudaSuccess ? LSA_OK : LSA_ERR_CUDA;
}
