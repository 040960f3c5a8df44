// Device-side FP8 quantisation arithmetic shared by the rowwise, per-channel
// and per-tensor kernels.
//
// For one scale S (a row's, a channel's or a tensor's):
//     S = fp32(amax) / fmax                (IEEE fp32 division; 1 for amax == 0)
//     q = RNEsat_fmt( RN_fp32(x / S) )     ("ComfyUI自定义节点开发适配Stable
//                                           Diffusion 3.5 FP8技术要点", section
//                                           "FP8：不只是精度减半", steps 2-3)
// RNEsat is cvt.rn.satfinite.{e4m3x2,e5m2x2}.f32: round to nearest, ties to
// even, magnitudes beyond the largest finite value clamp to it.
//
// The quotient RN_fp32(x / S) is the IEEE fp32 division. Dividing each
// element costs a reciprocal on the XU pipe plus several FMAs, which made the
// quantiser issue-bound. Instead each scale gets one correctly rounded
// reciprocal R = RN(1 / S) and every element takes Markstein's corrected
// quotient (P. Markstein, "Computation of elementary functions on the IBM
// RISC System/6000 processor", IBM J. Res. Develop. 34(1), 1990):
//     q0 = RN(x R);   e = x - q0 S  (one FMA, exact);   q = RN(q0 + e R)
// with the pair arithmetic done two lanes at a time (f32x2); each code takes
// its sign bit from x, which also fixes the sign of zero quotients. This path
// is taken only when amax >= 2^-64, so every x whose quotient can reach a
// nonzero FP8 code is a normal fp32 number; smaller amax takes the IEEE
// division. fp8dit_selftest_quotient() compares the resulting FP8 codes with
// the IEEE-division path for every pair (bf16 x, bf16 amax) with |x| <= amax,
// in both formats.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "fp8dit_internal.cuh"

namespace fp8dit {

template <int FMT>
struct Fp8Fmt;
template <>
struct Fp8Fmt<FP8DIT_E4M3FN> {
    static constexpr float kMax = 448.0f;
    static constexpr __nv_fp8_interpretation_t kInterp = __NV_E4M3;
};
template <>
struct Fp8Fmt<FP8DIT_E5M2> {
    static constexpr float kMax = 57344.0f;
    static constexpr __nv_fp8_interpretation_t kInterp = __NV_E5M2;
};

constexpr float kFastQuotientMinAmax = 0x1p-64f;

// Everything the element loop needs for one scale.
struct ScaleCtx {
    float s;     // the stored scale S
    float r;     // RN(1 / S), valid when fast
    bool fast;   // corrected-reciprocal quotient allowed
};

template <int FMT>
__device__ __forceinline__ ScaleCtx scale_ctx(float amax) {
    ScaleCtx c;
    c.s = amax == 0.0f ? 1.0f : __fdiv_rn(amax, Fp8Fmt<FMT>::kMax);
    c.fast = amax >= kFastQuotientMinAmax;
    c.r = __frcp_rn(c.s);
    return c;
}

// ---- packed fp32 pairs (sm_100a f32x2 arithmetic; each lane is an IEEE
// round-to-nearest multiply or fused multiply-add).
typedef unsigned long long f32x2_t;
__device__ __forceinline__ f32x2_t f2_pack(float lo, float hi) {
    f32x2_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float2 f2_unpack(f32x2_t v) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
    return make_float2(lo, hi);
}
__device__ __forceinline__ f32x2_t f2_mul(f32x2_t a, f32x2_t b) {
    f32x2_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ f32x2_t f2_fma(f32x2_t a, f32x2_t b, f32x2_t c) {
    f32x2_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// The per-scale operands of the packed quotient: {R, R} and {-S, -S}.
struct Quot2 {
    f32x2_t r2, ns2;
    float s;
};
__device__ __forceinline__ Quot2 quot2_of(const ScaleCtx& c) {
    return Quot2{f2_pack(c.r, c.r), f2_pack(-c.s, -c.s), c.s};
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// RN_fp32(x / S) for the two bf16 of w (low element first). FAST selects the
// corrected-reciprocal quotient; the IEEE division otherwise. The sign of a
// zero quotient may differ from x's; callers take the code's sign bit from x.
template <bool FAST>
__device__ __forceinline__ float2 quotient2(uint32_t w, const Quot2& q) {
    if (FAST) {
        const f32x2_t x2 = f2_pack(bf16_lo(w), bf16_hi(w));
        const f32x2_t q0 = f2_mul(x2, q.r2);
        const f32x2_t e = f2_fma(q0, q.ns2, x2);  // x - q0 S, exact
        return f2_unpack(f2_fma(e, q.r2, q0));
    }
    return make_float2(__fdiv_rn(bf16_lo(w), q.s), __fdiv_rn(bf16_hi(w), q.s));
}

// Two bf16 (one 32-bit word) -> two FP8 codes in the low 16 bits (low element first), sign bits not yet applied.
template <int FMT, bool FAST>
__device__ __forceinline__ uint32_t codes2(uint32_t w, const Quot2& q) {
    return (uint32_t)__nv_cvt_float2_to_fp8x2(quotient2<FAST>(w, q), __NV_SATFINITE, Fp8Fmt<FMT>::kInterp);
}

// Sign bits of the four bf16 in (w0, w1), placed in the sign bit of each code byte.
__device__ __forceinline__ uint32_t signs4(uint32_t w0, uint32_t w1) {
    return __byte_perm(w0, w1, 0x7531) & 0x80808080u;
}

// Eight bf16 (16 bytes) -> eight FP8 codes (8 bytes). Every code carries the
// sign of its input (x / S has x's sign, and zero quotients encode as a zero
// of that sign).
template <int FMT, bool FAST>
__device__ __forceinline__ uint2 quant8(const uint4& v, const Quot2& q) {
    uint2 o;
    o.x = (codes2<FMT, FAST>(v.x, q) | (codes2<FMT, FAST>(v.y, q) << 16)) | signs4(v.x, v.y);
    o.y = (codes2<FMT, FAST>(v.z, q) | (codes2<FMT, FAST>(v.w, q) << 16)) | signs4(v.z, v.w);
    return o;
}

// One bf16 -> one FP8 code (tails).
template <int FMT>
__device__ __forceinline__ uint8_t quant1(uint16_t b, const ScaleCtx& c) {
    const Quot2 q = quot2_of(c);
    const uint32_t w = (uint32_t)b;
    const uint32_t code = c.fast ? codes2<FMT, true>(w, q) : codes2<FMT, false>(w, q);
    return (uint8_t)((code & 0xffu) | ((b >> 8) & 0x80u));
}

// Running packed max of |bf16| over 2 / 8 values (sign bits cleared, then a
// bf16x2 max; non-negative bf16 order equals their bit-pattern order).
__device__ __forceinline__ uint32_t absmax2(uint32_t w, uint32_t acc) {
    __nv_bfloat162 a, b;
    *reinterpret_cast<uint32_t*>(&a) = acc;
    *reinterpret_cast<uint32_t*>(&b) = w & 0x7fff7fffu;
    a = __hmax2(a, b);
    return *reinterpret_cast<uint32_t*>(&a);
}
__device__ __forceinline__ uint32_t absmax8(const uint4& v, uint32_t acc) {
    return absmax2(v.w, absmax2(v.z, absmax2(v.y, absmax2(v.x, acc))));
}
// Larger of the two halves, as a 16-bit bf16 pattern.
__device__ __forceinline__ uint32_t fold_halves(uint32_t packed) { return max(packed & 0xffffu, packed >> 16); }
__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

}  // namespace fp8dit
