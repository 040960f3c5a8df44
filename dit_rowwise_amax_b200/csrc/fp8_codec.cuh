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
// and the sign of x is restored for quotients that round to zero. This path
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

// RN_fp32(x / S).
__device__ __forceinline__ float quotient(float x, const ScaleCtx& c) {
    if (c.fast) {
        const float q0 = __fmul_rn(x, c.r);
        const float e = __fmaf_rn(-q0, c.s, x);
        return copysignf(__fmaf_rn(e, c.r, q0), x);
    }
    return __fdiv_rn(x, c.s);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Two bf16 (one 32-bit word) -> two FP8 codes, low byte = low element.
template <int FMT>
__device__ __forceinline__ uint32_t quant2(uint32_t w, const ScaleCtx& c) {
    const float2 qf = make_float2(quotient(bf16_lo(w), c), quotient(bf16_hi(w), c));
    return (uint32_t)__nv_cvt_float2_to_fp8x2(qf, __NV_SATFINITE, Fp8Fmt<FMT>::kInterp);
}

// Eight bf16 (16 bytes) -> eight FP8 codes (8 bytes).
template <int FMT>
__device__ __forceinline__ uint2 quant8(const uint4& v, const ScaleCtx& c) {
    uint2 o;
    o.x = quant2<FMT>(v.x, c) | (quant2<FMT>(v.y, c) << 16);
    o.y = quant2<FMT>(v.z, c) | (quant2<FMT>(v.w, c) << 16);
    return o;
}

template <int FMT>
__device__ __forceinline__ uint8_t quant1(uint16_t b, const ScaleCtx& c) {
    const float q = quotient(__uint_as_float((uint32_t)b << 16), c);
    return (uint8_t)(__nv_cvt_float2_to_fp8x2(make_float2(q, 0.0f), __NV_SATFINITE, Fp8Fmt<FMT>::kInterp) & 0xffu);
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
