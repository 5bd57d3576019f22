/*
 * Seeded synthetic input generator.
 *
 * Serves both the fp64 CPU oracle and the CUDA path's tests and benchmark with
 * the SAME inputs: random-init weights, prompt tokens, precomputed prompt KV
 * caches and synthetic logits.  It holds none of the denoising method's
 * arithmetic -- only a counter-based hash and a fixed map from hash words to
 * numbers -- so that every element can be regenerated independently by
 * (seed, tensor id, element index) without storing a 50 GB file.
 *
 * Hash: the splitmix64 output function (Steele, Lea & Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014), applied to a Weyl sequence
 * key + (i+1)*gamma, so element i of a stream is one hash evaluation.
 *
 * Normal-ish values: Irwin-Hall sum of the four 16-bit fields of one word,
 *   z = (sum_j (u_j + 1/2) / 65536 - 2) * sqrt(3)   (mean 0, variance 1),
 * computed exactly in integers then scaled by one correctly rounded double
 * multiply, then rounded to bf16 (round to nearest even) by integer code.
 */
#include <stdint.h>
#include <string.h>
#include <math.h>

#define GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t id) {
    return mix64(mix64(seed + GAMMA) ^ (id * 0xD1B54A32D192ED03ULL + 0x8CB92BA72F3D8DD7ULL));
}

static inline uint64_t draw(uint64_t key, uint64_t i) { return mix64(key + (i + 1) * GAMMA); }

/* Irwin-Hall integer part: t = sum(u_j) + 2 - 131072, so z = t * sqrt(3) / 65536. */
static inline int64_t irwin_hall_t(uint64_t w) {
    int64_t s = (int64_t)(w & 0xFFFF) + (int64_t)((w >> 16) & 0xFFFF) +
                (int64_t)((w >> 32) & 0xFFFF) + (int64_t)(w >> 48);
    return s + 2 - 131072;
}

/* double -> bf16 bits, round to nearest even, directly from the double (no
 * intermediate float rounding).  Handles zero, normals and bf16 subnormals. */
static inline uint16_t bf16_bits_rne(double x) {
    uint64_t b;
    memcpy(&b, &x, 8);
    uint64_t sign = b >> 63;
    int ex = (int)((b >> 52) & 0x7FF);
    uint64_t man = b & ((1ULL << 52) - 1);
    if (ex == 0) return (uint16_t)(sign << 15); /* zero or double subnormal -> signed zero */
    if (ex == 0x7FF) return (uint16_t)((sign << 15) | 0x7F80 | (man ? 0x40 : 0));
    uint64_t m = man | (1ULL << 52);          /* 53-bit significand */
    int e = ex - 1023 + 127;                    /* bf16 biased exponent */
    int shift = 45;                             /* keep 8 significant bits */
    if (e <= 0) { shift += 1 - e; e = 0; }      /* bf16 subnormal */
    if (shift > 60) return (uint16_t)(sign << 15);
    uint64_t q = m >> shift;
    uint64_t rem = m & ((1ULL << shift) - 1);
    uint64_t half = 1ULL << (shift - 1);
    if (rem > half || (rem == half && (q & 1))) q++;
    uint64_t r;
    if (e == 0) {
        r = q;                                  /* q may reach 0x80: becomes the smallest normal */
    } else {
        if (q == 256) { q = 128; e++; }
        if (e >= 255) return (uint16_t)((sign << 15) | 0x7F80);
        r = ((uint64_t)e << 7) | (q & 0x7F);
    }
    return (uint16_t)((sign << 15) | r);
}

/* n values N(0, std^2)-like as bf16 bits, elements first..first+n-1 of stream (seed, id). */
void synth_normal_bf16(uint64_t seed, uint64_t id, uint64_t first, uint64_t n, double std,
                       uint16_t* out) {
    const uint64_t key = stream_key(seed, id);
    const double scale = std * (sqrt(3.0) / 65536.0);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i) {
        double x = (double)irwin_hall_t(draw(key, first + (uint64_t)i)) * scale;
        out[i] = bf16_bits_rne(x);
    }
}

/* Same values as fp32 (double rounded once to float). */
void synth_normal_f32(uint64_t seed, uint64_t id, uint64_t first, uint64_t n, double std,
                      float* out) {
    const uint64_t key = stream_key(seed, id);
    const double scale = std * (sqrt(3.0) / 65536.0);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i) {
        out[i] = (float)((double)irwin_hall_t(draw(key, first + (uint64_t)i)) * scale);
    }
}

/* Integers uniform in [0, V): high 32 bits of the word, multiply-shift. */
void synth_uniform_i32(uint64_t seed, uint64_t id, uint64_t first, uint64_t n, uint32_t V,
                       int32_t* out) {
    const uint64_t key = stream_key(seed, id);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i) {
        uint64_t hi = draw(key, first + (uint64_t)i) >> 32;
        out[i] = (int32_t)((hi * (uint64_t)V) >> 32);
    }
}

/* Raw 64-bit words (for tests of the generator itself). */
void synth_words(uint64_t seed, uint64_t id, uint64_t first, uint64_t n, uint64_t* out) {
    const uint64_t key = stream_key(seed, id);
    for (uint64_t i = 0; i < n; ++i) out[i] = draw(key, first + i);
}

/* Exposed for the generator's own unit tests. */
uint16_t synth_bf16_from_double(double x) { return bf16_bits_rne(x); }
