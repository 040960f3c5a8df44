// Per-token (rowwise) amax quantisation of bf16 rows to FP8 codes.
//
// Recipe ("ComfyUI自定义节点开发适配Stable Diffusion 3.5 FP8技术要点", section
// "FP8：不只是精度减半", steps 1-3, read for FP8): amax = max |x| over the row,
// S = amax / fmax (IEEE fp32 division; S = 1 for an all-zero row),
// q = RNE-saturating FP8 of the IEEE fp32 quotient x / S. Applied per token
// to activations ("从 BF16 到 FP8：HunyuanVideo1.5推理优化复盘", section 三.1)
// and per output channel to weights (section 二).
//
// Design: the op is HBM-bound (2 B read + 1 B written per element). A group
// of TPR threads owns one row and holds it in registers (VPT 16-byte vectors
// per thread, coalesced across the group), so each element is read from HBM
// exactly once: load -> packed bf16 |max| -> shuffle / shared-memory max across
// the group -> scale -> divide, convert two at a time with
// cvt.rn.satfinite.{e4m3x2,e5m2x2}.f32 -> 8-byte stores. Rows longer than
// 256 threads x 4 vectors x 8 = 8192 elements take a two-pass kernel whose
// second read of the row comes from L2.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "fp8dit_internal.cuh"

namespace fp8dit {
namespace {

template <int FMT>
struct Fmt;
template <>
struct Fmt<FP8DIT_E4M3FN> {
    static constexpr float kMax = 448.0f;
    static constexpr __nv_fp8_interpretation_t kInterp = __NV_E4M3;
};
template <>
struct Fmt<FP8DIT_E5M2> {
    static constexpr float kMax = 57344.0f;
    static constexpr __nv_fp8_interpretation_t kInterp = __NV_E5M2;
};

__device__ __forceinline__ __nv_bfloat162 as_bf162(uint32_t u) {
    __nv_bfloat162 r;
    *reinterpret_cast<uint32_t*>(&r) = u;
    return r;
}
__device__ __forceinline__ uint32_t as_u32(__nv_bfloat162 v) { return *reinterpret_cast<uint32_t*>(&v); }

// Running packed max of |bf16| over the 8 values of a 16-byte vector.
__device__ __forceinline__ uint32_t absmax8(const uint4& v, uint32_t acc) {
    __nv_bfloat162 m = as_bf162(acc);
    m = __hmax2(m, as_bf162(v.x & 0x7fff7fffu));
    m = __hmax2(m, as_bf162(v.y & 0x7fff7fffu));
    m = __hmax2(m, as_bf162(v.z & 0x7fff7fffu));
    m = __hmax2(m, as_bf162(v.w & 0x7fff7fffu));
    return as_u32(m);
}

// Larger of the two non-negative bf16 halves, as its 16-bit pattern.
__device__ __forceinline__ uint32_t fold_halves(uint32_t packed) {
    return max(packed & 0xffffu, packed >> 16);
}

template <int FMT>
__device__ __forceinline__ float scale_of(uint32_t amax_bits) {
    const float amax = __uint_as_float(amax_bits << 16);
    return amax == 0.0f ? 1.0f : __fdiv_rn(amax, Fmt<FMT>::kMax);
}

// Two bf16 (one 32-bit word) -> two FP8 codes (low byte = low element).
template <int FMT>
__device__ __forceinline__ uint32_t quant2(uint32_t w, float s) {
    const float lo = __uint_as_float(w << 16);
    const float hi = __uint_as_float(w & 0xffff0000u);
    float2 qf = make_float2(__fdiv_rn(lo, s), __fdiv_rn(hi, s));
    return (uint32_t)__nv_cvt_float2_to_fp8x2(qf, __NV_SATFINITE, Fmt<FMT>::kInterp);
}

template <int FMT>
__device__ __forceinline__ uint2 quant8(const uint4& v, float s) {
    uint2 o;
    o.x = quant2<FMT>(v.x, s) | (quant2<FMT>(v.y, s) << 16);
    o.y = quant2<FMT>(v.z, s) | (quant2<FMT>(v.w, s) << 16);
    return o;
}

constexpr int kThreads = 256;

// TPR threads per row (power of two, 8..256), VPT 16-byte vectors per thread.
template <int TPR, int VPT, int FMT>
__global__ void __launch_bounds__(kThreads) quantize_rows_regs(const uint16_t* __restrict__ x, int64_t M,
                                                                 int32_t K, int64_t ldx, uint8_t* __restrict__ q,
                                                                 int64_t ldq, float* __restrict__ scale) {
    constexpr int RPB = kThreads / TPR;
    const int t = threadIdx.x % TPR;
    const int r = threadIdx.x / TPR;
    const int64_t row = (int64_t)blockIdx.x * RPB + r;
    const bool active = row < M;
    const int nvec = K >> 3;
    const uint4* xr = reinterpret_cast<const uint4*>(x + (active ? row : 0) * ldx);

    uint4 v[VPT];
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int vi = i * TPR + t;
        v[i] = (active && vi < nvec) ? __ldcs(xr + vi) : make_uint4(0, 0, 0, 0);
    }
    uint32_t packed = 0;
#pragma unroll
    for (int i = 0; i < VPT; ++i) packed = absmax8(v[i], packed);
    uint32_t m = fold_halves(packed);

    if constexpr (TPR <= 32) {
#pragma unroll
        for (int off = TPR / 2; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
    } else {
        constexpr int WPR = TPR / 32;  // warps per row
        __shared__ uint32_t red[kThreads / 32];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
        __syncthreads();
        m = red[r * WPR];
#pragma unroll
        for (int w = 1; w < WPR; ++w) m = max(m, red[r * WPR + w]);
    }
    const float s = scale_of<FMT>(m);
    if (!active) return;

    uint8_t* qr = q + row * ldq;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int vi = i * TPR + t;
        if (vi < nvec) *reinterpret_cast<uint2*>(qr + (int64_t)vi * 8) = quant8<FMT>(v[i], s);
    }
    if (t == 0) scale[row] = s;
}

// One block per row (grid-strided): amax pass, then a quantise pass that
// re-reads the row (from L2). For rows beyond the register-resident kernel.
template <int FMT>
__global__ void __launch_bounds__(kThreads) quantize_rows_two_pass(const uint16_t* __restrict__ x, int64_t M,
                                                                     int64_t K, int64_t ldx,
                                                                     uint8_t* __restrict__ q, int64_t ldq,
                                                                     float* __restrict__ scale) {
    __shared__ uint32_t red[kThreads / 32];
    const int64_t nvec = K >> 3;
    for (int64_t row = blockIdx.x; row < M; row += gridDim.x) {
        const uint4* xr = reinterpret_cast<const uint4*>(x + row * ldx);
        uint32_t packed = 0;
        for (int64_t vi = threadIdx.x; vi < nvec; vi += kThreads) packed = absmax8(__ldg(xr + vi), packed);
        uint32_t m = fold_halves(packed);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
        __syncthreads();
        m = red[0];
#pragma unroll
        for (int w = 1; w < kThreads / 32; ++w) m = max(m, red[w]);
        __syncthreads();  // red is reused by the next row
        const float s = scale_of<FMT>(m);
        uint8_t* qr = q + row * ldq;
        for (int64_t vi = threadIdx.x; vi < nvec; vi += kThreads)
            *reinterpret_cast<uint2*>(qr + vi * 8) = quant8<FMT>(__ldcs(xr + vi), s);
        if (threadIdx.x == 0) scale[row] = s;
    }
}

template <int TPR, int VPT, int FMT>
cudaError_t launch_regs(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q, int64_t ldq,
                        float* scale, cudaStream_t stream) {
    constexpr int RPB = kThreads / TPR;
    const int64_t blocks = (M + RPB - 1) / RPB;
    if (blocks > 0x7fffffff) return cudaErrorInvalidConfiguration;
    quantize_rows_regs<TPR, VPT, FMT><<<(unsigned)blocks, kThreads, 0, stream>>>(x, M, (int32_t)K, ldx, q, ldq,
                                                                                  scale);
    return cudaGetLastError();
}

template <int FMT>
cudaError_t launch_fmt(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q, int64_t ldq,
                       float* scale, cudaStream_t stream, const DeviceInfo* dev) {
    const int64_t nvec = K / 8;
    if (nvec > 1024) {
        const int64_t grid = std::min<int64_t>(M, (int64_t)dev->num_sms * 8);
        quantize_rows_two_pass<FMT><<<(unsigned)grid, kThreads, 0, stream>>>(x, M, K, ldx, q, ldq, scale);
        return cudaGetLastError();
    }
    // Smallest power-of-two group (>= 8 threads) that covers the row with <= 4 vectors each.
    int tpr = 8;
    while (tpr * 4 < nvec) tpr *= 2;
    const bool two = nvec <= tpr * 2;
#define FP8DIT_Q_CASE(T)                                                                        \
    case T:                                                                                     \
        return two ? launch_regs<T, 2, FMT>(x, M, K, ldx, q, ldq, scale, stream)                \
                   : launch_regs<T, 4, FMT>(x, M, K, ldx, q, ldq, scale, stream);
    switch (tpr) {
        FP8DIT_Q_CASE(8)
        FP8DIT_Q_CASE(16)
        FP8DIT_Q_CASE(32)
        FP8DIT_Q_CASE(64)
        FP8DIT_Q_CASE(128)
        FP8DIT_Q_CASE(256)
        default:
            return cudaErrorInvalidValue;
    }
#undef FP8DIT_Q_CASE
}

}  // namespace

cudaError_t launch_quantize_rows(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int fmt, uint8_t* q,
                                 int64_t ldq, float* scale, cudaStream_t stream, const DeviceInfo* dev) {
    if (M == 0) return cudaSuccess;
    return fmt == FP8DIT_E4M3FN ? launch_fmt<FP8DIT_E4M3FN>(x, M, K, ldx, q, ldq, scale, stream, dev)
                                : launch_fmt<FP8DIT_E5M2>(x, M, K, ldx, q, ldq, scale, stream, dev);
}

}  // namespace fp8dit
