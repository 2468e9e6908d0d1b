/*
 * Seeded synthetic inputs for the MoE router gating workloads.
 *
 * This file generates numbers and nothing else: it holds none of the gating
 * arithmetic (no dot products, no selection, no softmax).  Both the CPU oracle
 * and the CUDA path consume the arrays it writes, so the two sides always see
 * bit-identical bf16 inputs.
 *
 * Generator: the SplitMix64 sequence (Steele, Lea and Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014).  For a tensor identified by
 * (seed, stream) the key is mix(mix(seed) ^ stream * C); the p-th 64-bit draw is
 * mix(key + (p + 1) * gamma).  Draw p feeds elements 2p and 2p+1 through the
 * Box-Muller transform (Box and Muller, 1958), so every element depends only on
 * (seed, stream, index): any slice of a tensor can be regenerated on its own,
 * in any order and on any number of threads, with the same result.
 *
 * Rounding to bf16: fp64 -> fp32 (round to nearest even, by the C cast) ->
 * bf16 (round to nearest even on the upper 16 bits).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define SYNTH_GAMMA 0x9E3779B97F4A7C15ULL
#define SYNTH_STREAM_MUL 0xD1B54A32D192ED03ULL

static inline uint64_t synth_mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static inline uint64_t synth_key(uint64_t seed, uint64_t stream) {
    return synth_mix64(synth_mix64(seed + SYNTH_GAMMA) ^ (stream * SYNTH_STREAM_MUL));
}

/* Standard normal deviate for element `index` of the tensor keyed by `key`. */
static inline double synth_normal_at(uint64_t key, int64_t index) {
    const uint64_t p = (uint64_t)index >> 1;
    const uint64_t r = synth_mix64(key + (p + 1) * SYNTH_GAMMA);
    const double u1 = ((double)(r >> 32) + 0.5) * (1.0 / 4294967296.0);  /* (0,1) */
    const double u2 = (double)(r & 0xFFFFFFFFULL) * (1.0 / 4294967296.0); /* [0,1) */
    const double rad = sqrt(-2.0 * log(u1));
    const double ang = 6.283185307179586476925286766559 * u2;
    return (index & 1) ? rad * sin(ang) : rad * cos(ang);
}

static inline uint16_t synth_bf16_rne(double v) {
    float f = (float)v;
    uint32_t bits;
    memcpy(&bits, &f, sizeof bits);
    if ((bits & 0x7F800000u) == 0x7F800000u && (bits & 0x007FFFFFu)) {
        return (uint16_t)((bits >> 16) | 0x0040u); /* quiet NaN */
    }
    bits += 0x7FFFu + ((bits >> 16) & 1u);
    return (uint16_t)(bits >> 16);
}

/* out[i] = normal(start + i) for i in [0, count), fp64. */
void synth_normal_f64(uint64_t seed, uint64_t stream, int64_t start, int64_t count, double* out) {
    const uint64_t key = synth_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) out[i] = synth_normal_at(key, start + i);
}

/* out[i] = bf16(scale * normal(start + i)). */
void synth_normal_bf16(uint64_t seed, uint64_t stream, int64_t start, int64_t count, double scale,
                       uint16_t* out) {
    const uint64_t key = synth_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) out[i] = synth_bf16_rne(scale * synth_normal_at(key, start + i));
}

/*
 * Rows [row0, row0 + nrows) of a [*, cols] tensor whose element (r, c) is
 * bf16(normal(r * cols + c) + alpha * vec[c]).  Used for hidden states with a
 * shared direction added to every token.
 */
void synth_normal_plus_vec_bf16(uint64_t seed, uint64_t stream, int64_t row0, int64_t nrows, int64_t cols,
                                const double* vec, double alpha, uint16_t* out) {
    const uint64_t key = synth_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < nrows; ++r) {
        const int64_t base = (row0 + r) * cols;
        for (int64_t c = 0; c < cols; ++c)
            out[r * cols + c] = synth_bf16_rne(synth_normal_at(key, base + c) + alpha * vec[c]);
    }
}

/* out[i] = bf16(in[i]). */
void synth_round_bf16(const double* in, int64_t count, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) out[i] = synth_bf16_rne(in[i]);
}
