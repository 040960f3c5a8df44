/*
 * CPU ORACLE — TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously correct restatement of what the FP8 DiT linear
 * path computes. Only the tests, the smoke check and the benchmark's CPU
 * baseline may load it; the product library never links or calls it, and
 * the two share no source, header, table or helper.
 *
 * Sources (page title, section):
 *  - "ComfyUI自定义节点开发适配Stable Diffusion 3.5 FP8技术要点", section
 *    "FP8：不只是精度减半": the E4M3 / E5M2 formats and the amax recipe
 *    (1) calibrate max|x|, (2) S = max|x| / fmax, (3) x_q = round(x / S),
 *    (4) x = x_q * S. The page writes fmax = 2^7 - 1 and "8-bit integer";
 *    both are read as the FP8 format's largest finite value and its code
 *    byte (448 for E4M3FN, 57344 for E5M2).
 *  - "从 BF16 到 FP8：HunyuanVideo1.5推理优化复盘", section 二 (weights
 *    quantised per output channel ahead of time, activations per token at
 *    run time) and section 三.1 (BF16 activation -> dynamic per-token FP8
 *    quant -> FP8 GEMM -> scale / bias / output dtype).
 *  - "Quantize Model to FP8 Format": whole state-dict tensors converted to
 *    float8_e4m3fn or float8_e5m2 with a scale (one scale per tensor); the
 *    tensors may be bf16, fp16 or fp32.
 *
 * Formats (OCP 8-bit floating point, which the pages name):
 *  E4M3FN: bias 7, normal (-1)^s 2^(e-7) (1 + m/8), subnormal (-1)^s 2^-6 m/8,
 *          S.1111.111 is NaN, no infinity, largest finite 448 (0x7E).
 *  E5M2:   bias 15, normal (-1)^s 2^(e-15) (1 + m/4), subnormal 2^-14 m/4,
 *          exponent 31 with m = 0 is infinity, m != 0 NaN, largest 57344.
 *
 * Readings where the pages are silent: encode rounds to the nearest code
 * with ties to the even mantissa and saturates to +-fmax; the scale and the
 * quotient are IEEE fp32 divisions (the page writes x / S); an all-zero row
 * or tensor gets S = 1; signs of zero and of underflowing values are kept.
 *
 * Build: gcc -O2 -fopenmp -fno-fast-math -ffp-contract=off (IEEE fp32
 * division with subnormals; no flush-to-zero).
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { OR_E4M3FN = 0, OR_E5M2 = 1 };

/* ------------------------------------------------------------ formats */
static int mant_bits(int fmt) { return fmt == OR_E4M3FN ? 3 : 2; }
static int exp_bias(int fmt) { return fmt == OR_E4M3FN ? 7 : 15; }
static double max_finite(int fmt) { return fmt == OR_E4M3FN ? 448.0 : 57344.0; }
static uint8_t max_code(int fmt) { return fmt == OR_E4M3FN ? 0x7E : 0x7B; }

/* Value of an FP8 code, from the closed form of the format. */
double or_decode(int fmt, uint8_t code) {
    int sign = code >> 7;
    int mb = mant_bits(fmt);
    int e = (code & 0x7F) >> mb;
    int m = code & ((1 << mb) - 1);
    double mag;
    if (fmt == OR_E4M3FN) {
        if (e == 15 && m == 7) return NAN;
        mag = (e == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    } else {
        if (e == 31) return m == 0 ? (sign ? -INFINITY : INFINITY) : NAN;
        mag = (e == 0) ? ldexp((double)m / 4.0, -14) : ldexp(1.0 + (double)m / 4.0, e - 15);
    }
    return sign ? -mag : mag;
}

/*
 * Nearest FP8 code to the fp32 value v: round half to even on the mantissa,
 * then clamp magnitudes above fmax to fmax. NaN maps to the NaN code with
 * v's sign; infinities saturate (outside the path's contract, kept for the
 * exhaustive encode report only).
 */
uint8_t or_encode(int fmt, float v) {
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    if (isnan(v)) return sign | 0x7F;
    double a = fabs((double)v);
    if (a >= max_finite(fmt)) return sign | max_code(fmt);
    int mb = mant_bits(fmt);
    int emin = 1 - exp_bias(fmt); /* exponent of the smallest normal */
    int e;                        /* a in [2^e, 2^(e+1)) for normal a */
    if (a < ldexp(1.0, emin)) {
        e = emin; /* subnormal range: the spacing is that of the smallest binade */
    } else {
        int fe;
        frexp(a, &fe); /* a = f * 2^fe with f in [0.5, 1) */
        e = fe - 1;
    }
    double quantum = ldexp(1.0, e - mb);
    double r = rint(a / quantum); /* exact division by a power of two; rint rounds half to even */
    if (r * quantum > max_finite(fmt)) return sign | max_code(fmt);
    uint8_t code;
    if (r * quantum < ldexp(1.0, emin)) {
        code = (uint8_t)r; /* subnormal: exponent field 0, mantissa r */
    } else {
        /* r in [2^mb, 2^(mb+1)]; r == 2^(mb+1) carries into the exponent. */
        int biased = e + exp_bias(fmt);
        code = (uint8_t)((biased << mb) + ((int)r - (1 << mb)));
    }
    return sign | code;
}

float or_bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* ---------------------------------------------------------- quantisers */
/* S = fp32(amax) / fmax as an IEEE fp32 division; S = 1 for amax == 0. */
static float scale_from_amax(int fmt, float amax) {
    return amax == 0.0f ? 1.0f : amax / (float)max_finite(fmt);
}

/* Per-row amax quantisation of bf16 x[M, K] (row stride ldx elements).
 * q[m, k] = encode(fp32(x[m, k]) / S[m]), q row stride ldq bytes. */
void or_quantize_rows(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int fmt,
                      uint8_t* q, int64_t ldq, float* s) {
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t* row = x + m * ldx;
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(or_bf16_to_f32(row[k]));
            if (a > amax) amax = a;
        }
        float sm = scale_from_amax(fmt, amax);
        s[m] = sm;
        for (int64_t k = 0; k < K; ++k) {
            float quotient = or_bf16_to_f32(row[k]) / sm;
            q[m * ldq + k] = or_encode(fmt, quotient);
        }
    }
}

/* Per-tensor amax quantisation: one scale for all n elements. */
void or_quantize_tensor(const uint16_t* x, int64_t n, int fmt, uint8_t* q, float* s) {
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(or_bf16_to_f32(x[i]));
        if (a > amax) amax = a;
    }
    float st = scale_from_amax(fmt, amax);
    *s = st;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) q[i] = or_encode(fmt, or_bf16_to_f32(x[i]) / st);
}

/*
 * fp16 bit pattern -> fp32, from the closed form of IEEE binary16: bias 15,
 * normal (-1)^s 2^(e-15) (1 + m/1024), subnormal (-1)^s 2^-14 m/1024,
 * exponent 31 is infinity (m = 0) or NaN. Every binary16 value is exact in fp32.
 */
float or_f16_to_f32(uint16_t h) {
    int sign = h >> 15;
    int e = (h >> 10) & 0x1F;
    int m = h & 0x3FF;
    double mag;
    if (e == 31) mag = m == 0 ? INFINITY : NAN;
    else if (e == 0) mag = ldexp((double)m / 1024.0, -14);
    else mag = ldexp(1.0 + (double)m / 1024.0, e - 15);
    return (float)(sign ? -mag : mag);
}

/* Element types a state-dict tensor may hold ("Quantize Model to FP8 Format":
 * the node converts the model's floating weights, whatever their precision). */
enum { OR_SRC_BF16 = 0, OR_SRC_F16 = 1, OR_SRC_F32 = 2 };

static float load_elem(int src, const void* x, int64_t i) {
    switch (src) {
        case OR_SRC_F16:
            return or_f16_to_f32(((const uint16_t*)x)[i]);
        case OR_SRC_F32:
            return ((const float*)x)[i];
        default:
            return or_bf16_to_f32(((const uint16_t*)x)[i]);
    }
}

/* Per-tensor amax quantisation of n elements of type src (each exact in fp32):
 * amax = max |x|, S = fp32(amax) / fmax, q = encode(x / S), as for bf16. */
void or_quantize_tensor_typed(const void* x, int src, int64_t n, int fmt, uint8_t* q, float* s) {
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(load_elem(src, x, i));
        if (a > amax) amax = a;
    }
    float st = scale_from_amax(fmt, amax);
    *s = st;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) q[i] = or_encode(fmt, load_elem(src, x, i) / st);
}

/* ---------------------------------------------------------- linear */
/*
 * Every E4M3FN value is an integer multiple of 2^-9 (the subnormal step),
 * with |integer| <= 448 * 2^9 < 2^18. A dot product of two such vectors is
 * therefore an integer multiple of 2^-18, and an int64 sum of the integer
 * products is exact for any K below 2^27.
 */
static void e4m3_units_table(int64_t units[256]) {
    for (int c = 0; c < 256; ++c) {
        double v = or_decode(OR_E4M3FN, (uint8_t)c);
        units[c] = isnan(v) ? 0 : (int64_t)(v * 512.0); /* NaN codes never leave a quantiser */
    }
}

/* y[m, n] = (sum_k A[m,k] W[n,k]) * sa[m] * sw[n] + bias[n], in double.
 * qa is [M, K] and qw is [N, K], both K-contiguous; bias may be NULL. */
static double linear_one(const int64_t units[256], const uint8_t* qa, const float* sa,
                         const uint8_t* qw, const float* sw, const uint16_t* bias, int64_t K,
                         int64_t m, int64_t n) {
    const uint8_t* a = qa + m * K;
    const uint8_t* w = qw + n * K;
    int64_t dot = 0;
    for (int64_t k = 0; k < K; ++k) dot += units[a[k]] * units[w[k]];
    double y = ldexp((double)dot, -18) * (double)sa[m] * (double)sw[n];
    if (bias) y += (double)or_bf16_to_f32(bias[n]);
    return y;
}

void or_linear(const uint8_t* qa, const float* sa, const uint8_t* qw, const float* sw,
               const uint16_t* bias, int64_t M, int64_t N, int64_t K, double* y) {
    int64_t units[256];
    e4m3_units_table(units);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) y[m * N + n] = linear_one(units, qa, sa, qw, sw, bias, K, m, n);
}

/* The same, at cnt listed (m, n) positions only. */
void or_linear_at(const uint8_t* qa, const float* sa, const uint8_t* qw, const float* sw,
                  const uint16_t* bias, int64_t K, const int64_t* ms, const int64_t* ns,
                  int64_t cnt, double* y) {
    int64_t units[256];
    e4m3_units_table(units);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < cnt; ++i) y[i] = linear_one(units, qa, sa, qw, sw, bias, K, ms[i], ns[i]);
}

/* Integer dot products sum_k units(A[m,k]) units(W[n,k]) for all (m, n): the
 * exact quantity behind or_linear, exposed so tests can pin it. */
void or_dot_units(const uint8_t* qa, const uint8_t* qw, int64_t M, int64_t N, int64_t K, int64_t* dot) {
    int64_t units[256];
    e4m3_units_table(units);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int64_t acc = 0;
            for (int64_t k = 0; k < K; ++k) acc += units[qa[m * K + k]] * units[qw[n * K + k]];
            dot[m * N + n] = acc;
        }
}

/* ----------------------------------------------------- FP8 weight-only linear */
/*
 * The FP8 weight-only configuration with scales, compared on the
 * longcat-avatar-compare page (section 速度总览): the activation stays bf16, only the weight is FP8
 * with its per-channel scale.
 *   y[m, n] = (sum_k A[m,k] dec(qw[n,k])) * sw[n] + bias[n], in double.
 * Every product of a bf16 value (8 significant bits) and an E4M3 value (4) is
 * exact in double; the sum is plain double accumulation in k order.
 */
void or_linear_weight_only(const uint16_t* a, const uint8_t* qw, const float* sw, const uint16_t* bias,
                           int64_t M, int64_t N, int64_t K, double* y) {
    double wv[256];
    for (int c = 0; c < 256; ++c) {
        double v = or_decode(OR_E4M3FN, (uint8_t)c);
        wv[c] = isnan(v) ? 0.0 : v;
    }
#pragma omp parallel
    {
        double* arow = (double*)malloc((size_t)K * sizeof(double)); /* row m of A as doubles (exact) */
#pragma omp for schedule(dynamic, 1)
        for (int64_t m = 0; m < M; ++m) {
            for (int64_t k = 0; k < K; ++k) arow[k] = (double)or_bf16_to_f32(a[m * K + k]);
            for (int64_t n = 0; n < N; ++n) {
                double dot = 0.0;
                for (int64_t k = 0; k < K; ++k) dot += arow[k] * wv[qw[n * K + k]];
                double v = dot * (double)sw[n];
                if (bias) v += (double)or_bf16_to_f32(bias[n]);
                y[m * N + n] = v;
            }
        }
        free(arow);
    }
}

/* ----------------------------------------------------- producer activations */
/*
 * "从 BF16 到 FP8：HunyuanVideo1.5推理优化复盘", section 三.5: the GELU / SiLU that
 * precedes FFN-down emits its output straight to FP8 with a per-token scale.
 * The activation is evaluated in double and rounded once to bf16; that bf16
 * tensor is what the rowwise recipe quantises.
 *   act 1: GELU, erf form   x Phi(x) = x/2 (1 + erf(x / sqrt 2)) = x/2 erfc(-x / sqrt 2)
 *   act 2: GELU, tanh form  x/2 (1 + tanh(u)) = x / (1 + exp(-2u)),
 *                           u = sqrt(2/pi) (x + 0.044715 x^3)
 *   act 3: SiLU             x / (1 + exp(-x))
 * The right-hand forms are the same functions without the cancellation of
 * 1 + erf / 1 + tanh for negative x.
 */
enum { OR_ACT_GELU_ERF = 1, OR_ACT_GELU_TANH = 2, OR_ACT_SILU = 3 };

double or_act(int act, double x) {
    switch (act) {
        case OR_ACT_GELU_ERF:
            return 0.5 * x * erfc(-x / sqrt(2.0));
        case OR_ACT_GELU_TANH:
            return x / (1.0 + exp(-2.0 * sqrt(2.0 / M_PI) * (x + 0.044715 * x * x * x)));
        case OR_ACT_SILU:
            return x / (1.0 + exp(-x));
        default:
            return x;
    }
}

/* Nearest bf16 to a double (ties to even), as a bit pattern; finite inputs
 * within the bf16 range. One rounding, straight from double. */
uint16_t or_round_bf16(double v) {
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0) return sign;
    int e;
    if (a < ldexp(1.0, -126)) {
        e = -126; /* subnormal bf16 spacing */
    } else {
        int fe;
        frexp(a, &fe);
        e = fe - 1;
    }
    double quantum = ldexp(1.0, e - 7);
    double r = rint(a / quantum) * quantum; /* representable in bf16, hence in fp32 */
    float f = (float)r;
    uint32_t u;
    memcpy(&u, &f, 4);
    return sign | (uint16_t)(u >> 16);
}

/* g[i] = bf16(act(h[i])) for n elements. */
void or_act_bf16(int act, const uint16_t* h, int64_t n, uint16_t* g) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) g[i] = or_round_bf16(or_act(act, (double)or_bf16_to_f32(h[i])));
}

/* Encode a batch of fp32 values (for codec tests). */
void or_encode_many(int fmt, const float* v, int64_t n, uint8_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = or_encode(fmt, v[i]);
}

/* Threads the oracle's parallel loops use (for reports). */
int or_num_threads(void) { return omp_get_max_threads(); }

/* Threads for the parallel loops that follow (timing the oracle single-threaded
   and on all cores); n <= 0 restores the default. */
void or_set_threads(int n) {
    static int default_threads = 0;
    if (default_threads == 0) default_threads = omp_get_max_threads();
    omp_set_num_threads(n > 0 ? n : default_threads);
}
