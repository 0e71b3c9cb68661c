/*
 * Seeded, counter-based synthetic input generator.
 *
 * This file holds no arithmetic of the TTT method: it only turns (seed, tensor tag,
 * element index) into pseudo-random numbers.  Both the CPU oracle and the CUDA path
 * consume the exact bits it produces (fp32 draws, optionally rounded to bf16 in the
 * Python wrapper).
 *
 * Generator: SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
 * generators", OOPSLA 2014), used counter-style: the i-th 64-bit draw of a stream is
 * mix64(key + (i + 1) * GOLDEN).  Normals come from the Box-Muller transform (cosine
 * branch only), one normal per pair of draws, so element i of a tensor depends on
 * nothing but (key, i) and any sub-range can be regenerated independently.
 */
#include <math.h>
#include <stdint.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static inline double unit_open(uint64_t x) {
    /* 53 random bits, centred in their bucket: strictly inside (0, 1). */
    return ((double)(x >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

/* Stream key of one tensor: two rounds of mixing over (seed, tag). */
uint64_t synth_stream_key(uint64_t seed, uint64_t tag) {
    return mix64(mix64(seed + GOLDEN) ^ (tag * 0xD1B54A32D192ED03ULL));
}

uint64_t synth_draw_u64(uint64_t key, uint64_t i) { return mix64(key + (i + 1) * GOLDEN); }

/* out[i] = (float)(mean + std * N_i), N_i standard normal from draws 2(first+i), 2(first+i)+1. */
void synth_normal_f32(uint64_t key, uint64_t first, int64_t n, double mean, double std,
                      float* out) {
    const double two_pi = 6.283185307179586476925286766559;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        uint64_t c = 2 * (first + (uint64_t)i);
        double u1 = unit_open(synth_draw_u64(key, c));
        double u2 = unit_open(synth_draw_u64(key, c + 1));
        double z = sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
        out[i] = (float)(mean + std * z);
    }
}

/* out[i] = (float)(logistic(N_i) / denom): the positive per-token rate distribution. */
void synth_logistic_normal_f32(uint64_t key, uint64_t first, int64_t n, double denom,
                               float* out) {
    const double two_pi = 6.283185307179586476925286766559;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        uint64_t c = 2 * (first + (uint64_t)i);
        double u1 = unit_open(synth_draw_u64(key, c));
        double u2 = unit_open(synth_draw_u64(key, c + 1));
        double z = sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
        out[i] = (float)((1.0 / (1.0 + exp(-z))) / denom);
    }
}
