/*
 * Seeded synthetic input generator (host C, OpenMP).
 *
 * This file holds no arithmetic of the attention method. It only draws the
 * random numbers that make up the synthetic workloads; the oracle and the
 * CUDA library both receive the same bytes from it.
 *
 * Generator: SplitMix64 (G. Steele, D. Lea, C. Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014), used counter-based: draw n of
 * a stream with key s is mix64(s + (n + 1) * GAMMA), i.e. the n-th output of a
 * SplitMix64 generator whose state starts at s. Every element is a pure
 * function of (key, index), so the fill is thread-count independent.
 *
 * Normals: Box-Muller (G. Box, M. Muller, 1958) on the two 32-bit halves of one
 * draw: u1 = (hi + 1) / 2^32 in (0, 1], u2 = lo / 2^32 in [0, 1),
 * z = sqrt(-2 ln u1) * cos(2 pi u2), evaluated in double with the host libm.
 */
#include <math.h>
#include <stdint.h>

#define GAMMA 0x9E3779B97F4A7C15ULL

uint64_t synth_mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* Stream key for (seed, a, b, c): chained mixing of the identifiers. */
uint64_t synth_key(uint64_t seed, uint64_t a, uint64_t b, uint64_t c) {
    uint64_t k = synth_mix64(seed + GAMMA);
    k = synth_mix64(k ^ ((a + 1) * GAMMA));
    k = synth_mix64(k ^ ((b + 1) * GAMMA));
    k = synth_mix64(k ^ ((c + 1) * GAMMA));
    return k;
}

static inline uint64_t draw(uint64_t key, uint64_t n) {
    return synth_mix64(key + (n + 1) * GAMMA);
}

static inline double normal_at(uint64_t key, uint64_t n) {
    uint64_t z = draw(key, n);
    double u1 = ((double)(z >> 32) + 1.0) * (1.0 / 4294967296.0);
    double u2 = (double)(z & 0xFFFFFFFFULL) * (1.0 / 4294967296.0);
    return sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
}

/* out[i] = RN_f32(normal(key, offset + i)), i < n. */
void synth_normals_f32(uint64_t key, uint64_t offset, int64_t n, float* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = (float)normal_at(key, offset + (uint64_t)i);
}

/* out[i] = normal(key, offset + i) in double, i < n. */
void synth_normals_f64(uint64_t key, uint64_t offset, int64_t n, double* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = normal_at(key, offset + (uint64_t)i);
}

/* out[i] = top 53 bits of draw(key, offset + i) / 2^53, in [0, 1). */
void synth_uniforms_f64(uint64_t key, uint64_t offset, int64_t n, double* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        out[i] = (double)(draw(key, offset + (uint64_t)i) >> 11) * (1.0 / 9007199254740992.0);
}

/* out[i] = draw(key, offset + i) (raw 64-bit words). */
void synth_words(uint64_t key, uint64_t offset, int64_t n, uint64_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = draw(key, offset + (uint64_t)i);
}

/*
 * Rows drawn per block: for row r (block j = r / L, clamped to nb - 1 for the
 * tail rows of a context that is not a multiple of L),
 *   out[r][c] = RN_f32(mu[j][c] + sigma[j] * normal(key, r * d + c)),
 * with mu + sigma * z evaluated in double.
 */
void synth_block_rows_f32(uint64_t key, const float* mu, const float* sigma, int64_t nb,
                          int64_t T, int64_t d, int64_t L, float* out) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < T; ++r) {
        int64_t j = r / L;
        if (j >= nb) j = nb - 1;
        const double s = (double)sigma[j];
        for (int64_t c = 0; c < d; ++c) {
            double z = normal_at(key, (uint64_t)(r * d + c));
            double v = (double)mu[j * d + c] + s * z;
            out[r * d + c] = (float)v;
        }
    }
}

/* Round float32 to bfloat16 bits, round to nearest, ties to even (finite inputs). */
void synth_f32_to_bf16(const float* in, int64_t n, uint16_t* out) {
    const uint32_t* u = (const uint32_t*)in;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        uint32_t b = u[i];
        uint32_t rounding = ((b >> 16) & 1u) + 0x7FFFu;
        out[i] = (uint16_t)((b + rounding) >> 16);
    }
}

/* Widen bfloat16 bits to float32 (exact). */
void synth_bf16_to_f32(const uint16_t* in, int64_t n, float* out) {
    uint32_t* u = (uint32_t*)out;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) u[i] = ((uint32_t)in[i]) << 16;
}
