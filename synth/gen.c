/*
 * Seeded, counter-based generator of synthetic inputs.
 *
 * This file draws random numbers only; it holds none of the arithmetic of the
 * sparse-attention method. It is shared by the CPU oracle, the tests and the
 * benchmark so that every side sees the same inputs.
 *
 * Definition (every element is independent, so any slice can be generated on
 * its own and in parallel):
 *   key(seed, id)  = mix(seed * 0x9E3779B97F4A7C15 + id + 1)
 *   word(i)        = mix(key + (i + 1) * 0x9E3779B97F4A7C15)
 *   mix(z)         = the SplitMix64 finaliser (Steele, Lea, Flood,
 *                    "Fast splittable pseudorandom number generators", 2014):
 *                    z ^= z>>30; z *= 0xBF58476D1CE4E5B9; z ^= z>>27;
 *                    z *= 0x94D049BB133111EB; z ^= z>>31
 *   uniform int in [lo, hi]: lo + word(i) mod (hi - lo + 1)
 *   standard normal (Box-Muller, fp64): u1 = ((word(2i) >> 11) + 0.5) / 2^53,
 *                    u2 = (word(2i+1) >> 11) / 2^53,
 *                    z = sqrt(-2 ln u1) * cos(2 pi u2)
 *   fp32 value  = z rounded to nearest-even fp32 (C conversion)
 *   bf16 value  = the fp32 value rounded to nearest-even bf16
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z ^= z >> 30;
    z *= 0xBF58476D1CE4E5B9ULL;
    z ^= z >> 27;
    z *= 0x94D049BB133111EBULL;
    z ^= z >> 31;
    return z;
}

static inline uint64_t stream_key(uint64_t seed, uint64_t id) {
    return mix64(seed * GOLDEN + id + 1);
}

static inline uint64_t word_at(uint64_t key, uint64_t i) {
    return mix64(key + (i + 1) * GOLDEN);
}

static inline double normal_at(uint64_t key, uint64_t i) {
    const double two53 = 9007199254740992.0;
    double u1 = ((double)(word_at(key, 2 * i) >> 11) + 0.5) / two53;
    double u2 = (double)(word_at(key, 2 * i + 1) >> 11) / two53;
    return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925286766559 * u2);
}

static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    uint32_t r = 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)((u + r) >> 16);
}

void synth_randint_i8(uint64_t seed, uint64_t id, int64_t start, int64_t n,
                      int32_t lo, int32_t hi, int8_t* out) {
    const uint64_t key = stream_key(seed, id);
    const uint64_t range = (uint64_t)((int64_t)hi - (int64_t)lo + 1);
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j)
        out[j] = (int8_t)(lo + (int64_t)(word_at(key, (uint64_t)(start + j)) % range));
}

void synth_randint_i32(uint64_t seed, uint64_t id, int64_t start, int64_t n,
                       int32_t lo, int32_t hi, int32_t* out) {
    const uint64_t key = stream_key(seed, id);
    const uint64_t range = (uint64_t)((int64_t)hi - (int64_t)lo + 1);
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j)
        out[j] = (int32_t)(lo + (int64_t)(word_at(key, (uint64_t)(start + j)) % range));
}

void synth_normal_f32(uint64_t seed, uint64_t id, int64_t start, int64_t n, float* out) {
    const uint64_t key = stream_key(seed, id);
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j)
        out[j] = (float)normal_at(key, (uint64_t)(start + j));
}

void synth_normal_bf16(uint64_t seed, uint64_t id, int64_t start, int64_t n, uint16_t* out) {
    const uint64_t key = stream_key(seed, id);
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j)
        out[j] = f32_to_bf16_rne((float)normal_at(key, (uint64_t)(start + j)));
}
