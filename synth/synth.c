/*
 * Seeded synthetic inputs for the FP8 DiT linear workloads.
 *
 * This module only draws random numbers and rounds them to bf16 bit
 * patterns. It holds none of the quantisation or GEMM arithmetic, so both
 * the CPU oracle and the CUDA path can consume the same bytes without
 * sharing any of the method's code.
 *
 * Generator: a counter-based stream. Element i of a stream with key k uses
 * the SplitMix64 finaliser (Steele, Lea, Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014) applied to
 * k + (i + 1) * 0x9e3779b97f4a7c15, and the top 53 bits become a double in
 * [0, 1). A standard normal for element i takes the Box-Muller transform
 * (cosine branch) of counters 2i and 2i+1. Outliers come from an
 * independent stream (key mixed with a constant): element i is an outlier
 * when its uniform is below p, and is then multiplied by a factor.
 * Every value is rounded double -> fp32 (RNE) -> bf16 (RNE).
 *
 * Output is identical for any thread count: each element depends only on
 * (key, i).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define SYNTH_GOLDEN 0x9e3779b97f4a7c15ULL
#define SYNTH_PI 3.14159265358979323846

static inline uint64_t sm64_finalise(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
    return z ^ (z >> 31);
}

static inline double sm64_u01(uint64_t key, uint64_t i) {
    uint64_t z = sm64_finalise(key + (i + 1) * SYNTH_GOLDEN);
    return (double)(z >> 11) * 0x1.0p-53;
}

static inline double sm64_normal(uint64_t key, uint64_t i) {
    double u1 = 1.0 - sm64_u01(key, 2 * i); /* (0, 1] keeps log finite */
    double u2 = sm64_u01(key, 2 * i + 1);
    return sqrt(-2.0 * log(u1)) * cos(2.0 * SYNTH_PI * u2);
}

/* double -> fp32 (RNE, the C conversion) -> bf16 (RNE on the bit pattern). */
static inline uint16_t to_bf16(double d) {
    float f = (float)d;
    uint32_t b;
    memcpy(&b, &f, 4);
    b += 0x7fffu + ((b >> 16) & 1u);
    return (uint16_t)(b >> 16);
}

/* Stream key from a seed and a tensor name (FNV-1a, then SplitMix64). */
uint64_t synth_key(uint64_t seed, const char* name) {
    uint64_t h = 0xcbf29ce484222325ULL;
    for (const unsigned char* p = (const unsigned char*)name; *p; ++p) {
        h ^= *p;
        h *= 0x100000001b3ULL;
    }
    return sm64_finalise(h ^ sm64_finalise(seed + SYNTH_GOLDEN));
}

/* out[i] = bf16(mean + std * z_i * (outlier_i ? factor : 1)). */
void synth_normal_bf16(uint64_t key, int64_t n, double mean, double std,
                       double outlier_p, double outlier_factor, uint16_t* out) {
    uint64_t okey = sm64_finalise(key ^ 0x6a09e667f3bcc909ULL);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double z = sm64_normal(key, (uint64_t)i);
        if (outlier_p > 0.0 && sm64_u01(okey, (uint64_t)i) < outlier_p) z *= outlier_factor;
        out[i] = to_bf16(mean + std * z);
    }
}

/* out[i] = bf16(GELU(z_i)), GELU(z) = z/2 * (1 + erf(z / sqrt 2)), in double. */
void synth_gelu_normal_bf16(uint64_t key, int64_t n, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double z = sm64_normal(key, (uint64_t)i);
        out[i] = to_bf16(0.5 * z * (1.0 + erf(z * 0.70710678118654752440)));
    }
}

/* Raw uniforms in [0,1), exposed for the generator's own tests. */
void synth_uniform(uint64_t key, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = sm64_u01(key, (uint64_t)i);
}
