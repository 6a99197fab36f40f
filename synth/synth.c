/*
 * Seeded synthetic inputs for the absorbed-MLA latent-cache attention path.
 *
 * This module holds no attention arithmetic. It only draws numbers: uniform
 * 64-bit words from a counter-based SplitMix64 stream (Steele, Lea and Flood,
 * "Fast splittable pseudorandom number generators", OOPSLA 2014), standard
 * normals by the Box-Muller transform (Box and Muller, 1958), integer ranges,
 * Fisher-Yates permutations and sorted samples without replacement.  Every
 * value is a pure function of (seed, stream, element index), so any slice of
 * a tensor can be regenerated on its own and the same bits feed both the GPU
 * path and the CPU oracle.  Floating-point draws are made in double precision
 * and rounded to bfloat16 with round-to-nearest-even.
 *
 * Built as a small shared library (gcc -O2 -fopenmp -shared -fPIC).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* State that starts the SplitMix64 sequence of (seed, stream). */
static inline uint64_t stream_key(uint64_t seed, uint64_t stream) {
    return mix64(seed * GOLDEN + 0x632BE59BD9B4E019ULL) ^ mix64(stream + 0xD1B54A32D192ED03ULL);
}

/* i-th output of the SplitMix64 sequence started at `key` (i >= 0). */
static inline uint64_t word_at(uint64_t key, uint64_t i) { return mix64(key + (i + 1) * GOLDEN); }

/* Uniform double in (0, 1]: 53 high bits of the word, shifted off zero. */
static inline double unit_at(uint64_t key, uint64_t i) {
    return (double)((word_at(key, i) >> 11) + 1) * (1.0 / 9007199254740992.0);
}

static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)((u >> 16) | ((u & 0xFFFF) ? 0x40 : 0));
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* Normal draw for element e: pair k = e/2 uses uniforms 2k and 2k+1; even
 * elements take the cosine branch, odd ones the sine branch. */
static inline double normal_at(uint64_t key, uint64_t e) {
    uint64_t k = e >> 1;
    double u1 = unit_at(key, 2 * k), u2 = unit_at(key, 2 * k + 1);
    double r = sqrt(-2.0 * log(u1));
    double t = 6.283185307179586476925286766559 * u2;
    return (e & 1) ? r * sin(t) : r * cos(t);
}

/* out[i] = bf16(std * N(0,1) draw of element offset+i), i in [0, n). */
void synth_normal_bf16(uint16_t *out, int64_t n, uint64_t seed, uint64_t stream, double std, int64_t offset) {
    uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double z = std * normal_at(key, (uint64_t)(offset + i));
        out[i] = f32_to_bf16_rne((float)z);
    }
}

/* Same draws, kept in double (used only to test the generator itself). */
void synth_normal_f64(double *out, int64_t n, uint64_t seed, uint64_t stream, double std, int64_t offset) {
    uint64_t key = stream_key(seed, stream);
    for (int64_t i = 0; i < n; ++i) out[i] = std * normal_at(key, (uint64_t)(offset + i));
}

/* out[i] = uniform integer in [lo, hi] (inclusive) for element offset+i. */
void synth_uniform_int(int64_t *out, int64_t n, uint64_t seed, uint64_t stream, int64_t lo, int64_t hi, int64_t offset) {
    uint64_t key = stream_key(seed, stream);
    double span = (double)(hi - lo + 1);
    for (int64_t i = 0; i < n; ++i) {
        double u = unit_at(key, (uint64_t)(offset + i)); /* (0,1] */
        int64_t v = lo + (int64_t)floor((1.0 - u) * span); /* [0,1) * span */
        if (v > hi) v = hi;
        out[i] = v;
    }
}

/* Fisher-Yates shuffle of 0..n-1 (Durstenfeld's in-place form). */
void synth_permutation(int32_t *out, int64_t n, uint64_t seed, uint64_t stream) {
    uint64_t key = stream_key(seed, stream);
    for (int64_t i = 0; i < n; ++i) out[i] = (int32_t)i;
    for (int64_t i = n - 1; i > 0; --i) {
        double u = unit_at(key, (uint64_t)(n - 1 - i));
        int64_t j = (int64_t)floor((1.0 - u) * (double)(i + 1));
        if (j > i) j = i;
        int32_t t = out[i];
        out[i] = out[j];
        out[j] = t;
    }
}

static int cmp_i32(const void *a, const void *b) {
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/* k distinct values from [0, range), sorted ascending: the first k slots of a
 * partial Fisher-Yates shuffle of 0..range-1.  `scratch` holds range ints. */
int synth_sorted_sample(int32_t *out, int64_t k, int64_t range, uint64_t seed, uint64_t stream, int32_t *scratch) {
    if (k < 0 || k > range) return -1;
    uint64_t key = stream_key(seed, stream);
    for (int64_t i = 0; i < range; ++i) scratch[i] = (int32_t)i;
    for (int64_t i = 0; i < k; ++i) {
        double u = unit_at(key, (uint64_t)i);
        int64_t j = i + (int64_t)floor((1.0 - u) * (double)(range - i));
        if (j >= range) j = range - 1;
        int32_t t = scratch[i];
        scratch[i] = scratch[j];
        scratch[j] = t;
    }
    memcpy(out, scratch, (size_t)k * sizeof(int32_t));
    qsort(out, (size_t)k, sizeof(int32_t), cmp_i32);
    return 0;
}

/* Raw words, for generator self-tests. */
void synth_words(uint64_t *out, int64_t n, uint64_t seed, uint64_t stream, int64_t offset) {
    uint64_t key = stream_key(seed, stream);
    for (int64_t i = 0; i < n; ++i) out[i] = word_at(key, (uint64_t)(offset + i));
}
