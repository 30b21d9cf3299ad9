/*
 * Seeded synthetic inputs, host side (plain C + OpenMP).
 *
 * This file holds no arithmetic of the mixture-of-experts method: it only
 * produces the random activations and weights that the oracle and the CUDA
 * path both consume.  A CUDA twin (synth_cuda.cu) implements the same
 * generator from the same definition so that large weight banks can be made
 * directly in device memory; the two are required to agree bit for bit.
 *
 * Definition (both twins implement exactly this):
 *   mix64(z)      = SplitMix64 output finaliser (Steele, Lea, Flood 2014):
 *                   z ^= z>>30; z *= 0xBF58476D1CE4E5B9;
 *                   z ^= z>>27; z *= 0x94D049BB133111EB; z ^= z>>31
 *   sm64(s, i)    = mix64(s + (i+1) * 0x9E3779B97F4A7C15)
 *                   (the i-th output of a SplitMix64 stream seeded with s)
 *   key(seed, tensor, layer) = sm64(seed, (tensor << 32) | layer)
 *   normal(key, j): take the 12 16-bit fields k_0..k_11 of
 *                   sm64(key,3j), sm64(key,3j+1), sm64(key,3j+2)
 *                   (low field first), n = sum(k_q) + 6 - 6*65536,
 *                   z = n / 65536 (exact in fp32): the Irwin-Hall sum of
 *                   twelve centred uniforms, an approximate N(0,1) bounded
 *                   by +-6.
 *   value_bf16    = bf16_rne( fp32_rne(z * sigma) )
 *
 * Every step is integer arithmetic or one correctly rounded IEEE fp32
 * multiply, so any conforming implementation yields identical bits.
 */
#include <stdint.h>
#include <string.h>

#define SM64_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static inline uint64_t sm64(uint64_t s, uint64_t i) {
    return mix64(s + (i + 1ULL) * SM64_GAMMA);
}

uint64_t synth_key(uint64_t seed, uint32_t tensor_id, uint32_t layer) {
    return sm64(seed, ((uint64_t)tensor_id << 32) | (uint64_t)layer);
}

uint64_t synth_u64(uint64_t key, uint64_t i) { return sm64(key, i); }

static inline float irwin_hall12(uint64_t key, uint64_t j) {
    uint64_t w[3];
    w[0] = sm64(key, 3 * j);
    w[1] = sm64(key, 3 * j + 1);
    w[2] = sm64(key, 3 * j + 2);
    int32_t s = 0;
    for (int a = 0; a < 3; ++a)
        for (int q = 0; q < 4; ++q) s += (int32_t)((w[a] >> (16 * q)) & 0xFFFFu);
    int32_t n = s + 6 - 6 * 65536;
    return (float)n * (1.0f / 65536.0f);
}

static inline uint16_t f32_to_bf16_rne(float v) {
    uint32_t u;
    memcpy(&u, &v, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40u);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* out[i] = bf16(normal(key, offset + i) * sigma), i in [0, n). */
void synth_normal_bf16(uint64_t key, uint64_t offset, uint64_t n, float sigma, uint16_t* out) {
    int64_t nn = (int64_t)n;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nn; ++i) {
        float z = irwin_hall12(key, offset + (uint64_t)i);
        float v = z * sigma;
        out[i] = f32_to_bf16_rne(v);
    }
}

/* out[i] = fp32(normal(key, offset + i) * sigma) (no bf16 rounding). */
void synth_normal_f32(uint64_t key, uint64_t offset, uint64_t n, float sigma, float* out) {
    int64_t nn = (int64_t)n;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nn; ++i) {
        float z = irwin_hall12(key, offset + (uint64_t)i);
        out[i] = z * sigma;
    }
}
