/*
 * Seeded synthetic inputs for the ragged / prefix-shared / tiered paged decode workloads.
 *
 * This file holds random draws only: counter-based SplitMix64 streams, uniform integers,
 * Box-Muller normals rounded to bf16, and Fisher-Yates permutations. It holds none of the
 * attention method's arithmetic (no retained-length rule, no grouping, no allocation, no
 * quantisation, no softmax). Both the CUDA path and the CPU oracle receive its bytes.
 *
 * Generator: SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
 * generators", OOPSLA 2014). Stream s of seed k has state  key(k, s) + (i + 1) * gamma  at
 * index i, and its i-th draw is the SplitMix64 output function applied to that state.
 * Every value is therefore a pure function of (seed, stream, index).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define SYNTH_GAMMA 0x9E3779B97F4A7C15ULL

static uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static uint64_t stream_key(uint64_t seed, uint64_t stream) {
    return mix64(seed ^ mix64(stream * SYNTH_GAMMA + 0x632BE59BD9B4E019ULL));
}

/* The SplitMix64 state from which stream s of seed k starts: draw i of the stream is the
 * (i+1)-th output of SplitMix64 seeded with this value. */
uint64_t synth_stream_key(uint64_t seed, uint64_t stream) { return stream_key(seed, stream); }

uint64_t synth_draw(uint64_t seed, uint64_t stream, uint64_t i) {
    return mix64(stream_key(seed, stream) + (i + 1) * SYNTH_GAMMA);
}

void synth_draws(uint64_t seed, uint64_t stream, uint64_t i0, int64_t n, uint64_t *out) {
    uint64_t key = stream_key(seed, stream);
    for (int64_t j = 0; j < n; ++j) out[j] = mix64(key + (i0 + (uint64_t)j + 1) * SYNTH_GAMMA);
}

/* Uniform integer in [lo, hi] (inclusive): lo + draw mod (hi - lo + 1). */
void synth_uniform_int(uint64_t seed, uint64_t stream, uint64_t i0, int64_t n, int64_t lo,
                       int64_t hi, int32_t *out) {
    uint64_t key = stream_key(seed, stream);
    uint64_t span = (uint64_t)(hi - lo + 1);
    for (int64_t j = 0; j < n; ++j)
        out[j] = (int32_t)(lo + (int64_t)(mix64(key + (i0 + (uint64_t)j + 1) * SYNTH_GAMMA) % span));
}

/* Round a float to bf16 bits, round-to-nearest-even; NaN stays a quiet NaN. */
static uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* Normal N(mean, sd^2) element i of a stream, from draws 2i and 2i+1 (Box-Muller, cosine
 * branch): u1 in (0, 1], u2 in [0, 1), both 53-bit. */
static double normal_at(uint64_t key, uint64_t i) {
    uint64_t a = mix64(key + (2 * i + 1) * SYNTH_GAMMA);
    uint64_t b = mix64(key + (2 * i + 2) * SYNTH_GAMMA);
    double u1 = ((double)(a >> 11) + 1.0) * (1.0 / 9007199254740992.0);
    double u2 = (double)(b >> 11) * (1.0 / 9007199254740992.0);
    return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925 * u2);
}

/* n normals (elements i0 .. i0+n-1 of the stream), scaled by sd and shifted by mean in
 * double, rounded to float and then to bf16 (RNE). Parallel over elements. */
void synth_normal_bf16(uint64_t seed, uint64_t stream, uint64_t i0, int64_t n, double mean,
                       double sd, uint16_t *out) {
    uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j)
        out[j] = f32_to_bf16_rne((float)(mean + sd * normal_at(key, i0 + (uint64_t)j)));
}

/* The same normals as doubles (no rounding), for small reference constructions. */
void synth_normal_f64(uint64_t seed, uint64_t stream, uint64_t i0, int64_t n, double *out) {
    uint64_t key = stream_key(seed, stream);
    for (int64_t j = 0; j < n; ++j) out[j] = normal_at(key, i0 + (uint64_t)j);
}

/* Fisher-Yates shuffle of 0 .. n-1: for i = n-1 down to 1, swap a[i] with a[j],
 * j = draw(n-1-i) mod (i+1). */
void synth_permutation(uint64_t seed, uint64_t stream, int64_t n, int32_t *out) {
    uint64_t key = stream_key(seed, stream);
    for (int64_t i = 0; i < n; ++i) out[i] = (int32_t)i;
    for (int64_t i = n - 1; i >= 1; --i) {
        uint64_t r = mix64(key + ((uint64_t)(n - 1 - i) + 1) * SYNTH_GAMMA);
        int64_t j = (int64_t)(r % (uint64_t)(i + 1));
        int32_t t = out[i];
        out[i] = out[j];
        out[j] = t;
    }
}
