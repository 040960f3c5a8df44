/*
 * CPU check of the corrected-reciprocal quotient the GPU quantisers use in
 * place of an IEEE fp32 division (Markstein, IBM J. Res. Develop. 34(1),
 * 1990): with S = amax / fmax and R = 1 / S (both IEEE fp32 divisions),
 *     q0 = x * R;  e = fma(-q0, S, x);  q = copysign(fma(e, R, q0), x)
 * for amax >= 2^-64. For every finite positive bf16 amax and every bf16 x
 * with |x| <= amax, q must equal the IEEE quotient x / S bit for bit, except
 * where both are below `zero_below` with the same sign (they then encode to
 * the same signed-zero FP8 code). Test infrastructure: not part of the
 * library or the oracle.
 *
 * Build: gcc -O2 -fopenmp -fno-fast-math -ffp-contract=off (separate
 * rounding of x * R; fmaf is the fused operation).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static float bf16(uint32_t b) {
    uint32_t u = b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static uint32_t bits(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    return u;
}

/* Returns pairs whose results would encode differently; *differ counts all
 * fp32 differences (informational). */
long long quotient_identity_check(float fmax, float zero_below, long long* differ) {
    long long bad = 0, diff = 0;
#pragma omp parallel for reduction(+ : bad, diff) schedule(dynamic, 64)
    for (uint32_t a = 1; a <= 0x7F7Fu; ++a) {
        const float amax = bf16(a);
        const float s = amax / fmax;
        const float r = 1.0f / s;
        const int fast = amax >= 0x1p-64f;
        for (uint32_t m = 0; m <= a; ++m) {
            for (uint32_t sg = 0; sg < 2; ++sg) {
                const float x = bf16(m | (sg << 15));
                const float qi = x / s;
                float qf = qi;
                if (fast) {
                    const float q0 = x * r;
                    const float e = fmaf(-q0, s, x);
                    qf = copysignf(fmaf(e, r, q0), x);
                }
                if (bits(qi) != bits(qf)) {
                    ++diff;
                    if (!(fabsf(qi) < zero_below && fabsf(qf) < zero_below && signbit(qi) == signbit(qf))) ++bad;
                }
            }
        }
    }
    *differ = diff;
    return bad;
}
