/* normal_host.c - host implementation of the seeded input generator defined in
 * datagen/__init__.py (counter-based SplitMix64, Irwin-Hall sum of twelve 16-bit
 * uniforms), for regenerating large slices of the K/V caches quickly on the CPU.
 * Input generation only: no arithmetic of the LSA method lives here. The numpy
 * definition in datagen/__init__.py is the reference; tests compare the two bit
 * for bit. */
#include <stdint.h>
#include <string.h>

#define DG_API __attribute__((visibility("default")))

static const uint64_t kGamma = 0x9E3779B97F4A7C15ull;

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

static inline float normal_at(uint64_t key, uint64_t idx) {
    int32_t acc = 0;
    for (int j = 0; j < 3; ++j) {
        const uint64_t w = mix64(key + (3ull * idx + (uint64_t)(j + 1)) * kGamma);
        acc += (int32_t)(w & 0xFFFFu) + (int32_t)((w >> 16) & 0xFFFFu) + (int32_t)((w >> 32) & 0xFFFFu) +
               (int32_t)(w >> 48);
    }
    return (float)(acc - 393210) * (1.0f / 65536.0f);
}

/* float32 -> bfloat16 (nearest-even) -> float32, for finite inputs. */
static inline float round_bf16(float x) {
    uint32_t u;
    memcpy(&u, &x, 4);
    u += 0x7FFFu + ((u >> 16) & 1u);
    u &= 0xFFFF0000u;
    float y;
    memcpy(&y, &u, 4);
    return y;
}

/* x_{idx[i]} for i < n. */
DG_API void dg_normal_f32(uint32_t seed, uint32_t tensor_id, const uint64_t *idx, int64_t n, float *out) {
    const uint64_t key = mix64(((uint64_t)seed << 32) | tensor_id);
    for (int64_t i = 0; i < n; ++i) out[i] = normal_at(key, idx[i]);
}

/* Rows of a cache [rows][H][Dh]: out[t][h][d] = x_{(tokens[t]*H + heads[h])*Dh + d}, rounded
 * through bfloat16 when bf16 != 0, as exact float32 values. */
DG_API void dg_cache_rows(uint32_t seed, uint32_t tensor_id, int64_t H, int64_t Dh, const int64_t *tokens,
                          int64_t ntok, const int64_t *heads, int64_t nheads, int bf16, float *out) {
    const uint64_t key = mix64(((uint64_t)seed << 32) | tensor_id);
    for (int64_t t = 0; t < ntok; ++t) {
        for (int64_t h = 0; h < nheads; ++h) {
            const uint64_t base = ((uint64_t)tokens[t] * (uint64_t)H + (uint64_t)heads[h]) * (uint64_t)Dh;
            float *o = out + (t * nheads + h) * Dh;
            for (int64_t d = 0; d < Dh; ++d) {
                const float x = normal_at(key, base + (uint64_t)d);
                o[d] = bf16 ? round_bf16(x) : x;
            }
        }
    }
}
