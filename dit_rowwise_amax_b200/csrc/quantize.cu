// Per-token (rowwise) amax quantisation of bf16 rows to FP8 codes.
//
// Recipe ("ComfyUI自定义节点开发适配Stable Diffusion 3.5 FP8技术要点", section
// "FP8：不只是精度减半", steps 1-3, read for FP8): amax = max |x| over the row,
// S = amax / fmax (IEEE fp32 division; S = 1 for an all-zero row),
// q = RNE-saturating FP8 of the fp32 quotient x / S. Applied per token to
// activations ("从 BF16 到 FP8：HunyuanVideo1.5推理优化复盘", section 三.1) and per
// output channel to weights (section 二).
//
// Design: the op is HBM-bound (2 B read + 1 B written per element). A group
// of TPR threads owns one row and holds it in registers (VPT 16-byte vectors
// per thread, coalesced across the group), so each element is read from HBM
// once: load -> packed bf16 |max| -> shuffle / shared-memory max across the
// group -> scale and reciprocal -> corrected-reciprocal quotient -> convert
// two at a time -> 8-byte stores. Blocks are persistent (grid = resident
// blocks) and load the next row group's vectors before quantising the
// current one, so HBM reads overlap the arithmetic. Rows longer than
// 256 threads x 4 vectors x 8 = 8192 elements take a two-pass kernel whose
// second read of the row comes from L2.
#include <algorithm>

#include "fp8_codec.cuh"

namespace fp8dit {
namespace {

constexpr int kThreads = 256;

template <int TPR, int VPT>
__device__ __forceinline__ void load_group(const uint16_t* __restrict__ x, int64_t M, int nvec, int64_t ldx,
                                           int64_t g, uint4 (&v)[VPT]) {
    constexpr int RPB = kThreads / TPR;
    const int t = threadIdx.x % TPR;
    const int64_t row = g * RPB + threadIdx.x / TPR;
    const bool active = row < M;
    const uint4* xr = reinterpret_cast<const uint4*>(x + (active ? row : 0) * ldx);
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int vi = i * TPR + t;
        v[i] = (active && vi < nvec) ? __ldcs(xr + vi) : make_uint4(0, 0, 0, 0);
    }
}

// TPR threads per row (power of two, 8..256), VPT 16-byte vectors per thread.
template <int TPR, int VPT, int FMT>
__global__ void __launch_bounds__(kThreads) quantize_rows_regs(const uint16_t* __restrict__ x, int64_t M,
                                                                 int32_t K, int64_t ldx, uint8_t* __restrict__ q,
                                                                 int64_t ldq, float* __restrict__ scale,
                                                                 int64_t groups) {
    constexpr int RPB = kThreads / TPR;
    constexpr int WPR = TPR / 32;  // warps per row (when TPR >= 32)
    __shared__ uint32_t red[2][kThreads / 32];
    const int t = threadIdx.x % TPR;
    const int r = threadIdx.x / TPR;
    const int nvec = K >> 3;

    uint4 cur[VPT], nxt[VPT];
    int64_t g = blockIdx.x;
    pdl_wait();  // x may be the previous kernel's output; q and scale its input
    pdl_trigger();
    load_group<TPR, VPT>(x, M, nvec, ldx, g, cur);
    for (int it = 0; g < groups; g += gridDim.x, ++it) {
        const int64_t gn = g + gridDim.x;
        if (gn < groups) load_group<TPR, VPT>(x, M, nvec, ldx, gn, nxt);

        uint32_t packed = 0;
#pragma unroll
        for (int i = 0; i < VPT; ++i) packed = absmax8(cur[i], packed);
        uint32_t m = fold_halves(packed);
        if constexpr (TPR <= 32) {
#pragma unroll
            for (int off = TPR / 2; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
        } else {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
            uint32_t* rb = red[it & 1];  // alternate buffers: no second barrier per group
            if ((threadIdx.x & 31) == 0) rb[threadIdx.x >> 5] = m;
            __syncthreads();
            m = rb[r * WPR];
#pragma unroll
            for (int w = 1; w < WPR; ++w) m = max(m, rb[r * WPR + w]);
        }
        const ScaleCtx c = scale_ctx<FMT>(bf16_bits_to_float(m));
        const int64_t row = g * RPB + r;
        if (row < M) {
            const Quot2 q2 = quot2_of(c);
            uint8_t* qr = q + row * ldq;
            if (c.fast) {
#pragma unroll
                for (int i = 0; i < VPT; ++i) {
                    const int vi = i * TPR + t;
                    if (vi < nvec) *reinterpret_cast<uint2*>(qr + (int64_t)vi * 8) = quant8<FMT, true>(cur[i], q2);
                }
            } else {
#pragma unroll
                for (int i = 0; i < VPT; ++i) {
                    const int vi = i * TPR + t;
                    if (vi < nvec) *reinterpret_cast<uint2*>(qr + (int64_t)vi * 8) = quant8<FMT, false>(cur[i], q2);
                }
            }
            if (t == 0) scale[row] = c.s;
        }
#pragma unroll
        for (int i = 0; i < VPT; ++i) cur[i] = nxt[i];
    }
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
    pdl_wait();
    pdl_trigger();
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
        const ScaleCtx c = scale_ctx<FMT>(bf16_bits_to_float(m));
        const Quot2 q2 = quot2_of(c);
        uint8_t* qr = q + row * ldq;
        if (c.fast) {
            for (int64_t vi = threadIdx.x; vi < nvec; vi += kThreads)
                *reinterpret_cast<uint2*>(qr + vi * 8) = quant8<FMT, true>(__ldcs(xr + vi), q2);
        } else {
            for (int64_t vi = threadIdx.x; vi < nvec; vi += kThreads)
                *reinterpret_cast<uint2*>(qr + vi * 8) = quant8<FMT, false>(__ldcs(xr + vi), q2);
        }
        if (threadIdx.x == 0) scale[row] = c.s;
    }
}

template <int TPR, int VPT, int FMT>
cudaError_t launch_regs(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q, int64_t ldq,
                        float* scale, cudaStream_t stream, const DeviceInfo* dev) {
    constexpr int RPB = kThreads / TPR;
    static int per_sm = 0;  // resident blocks per SM (same on every sm_100a device)
    if (per_sm == 0) {
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quantize_rows_regs<TPR, VPT, FMT>,
                                                                       kThreads, 0);
        if (e != cudaSuccess) return e;
        if (per_sm < 1) per_sm = 1;
    }
    const int64_t groups = (M + RPB - 1) / RPB;
    const int64_t grid = std::min<int64_t>(groups, (int64_t)dev->num_sms * per_sm);
    return launch_pdl(quantize_rows_regs<TPR, VPT, FMT>, dim3((unsigned)grid), dim3(kThreads), 0, stream, 1, x, M,
                      (int32_t)K, ldx, q, ldq, scale, groups);
}

template <int FMT>
cudaError_t launch_fmt(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q, int64_t ldq,
                       float* scale, cudaStream_t stream, const DeviceInfo* dev) {
    const int64_t nvec = K / 8;
    if (nvec > 1024) {
        const int64_t grid = std::min<int64_t>(M, (int64_t)dev->num_sms * 8);
        return launch_pdl(quantize_rows_two_pass<FMT>, dim3((unsigned)grid), dim3(kThreads), 0, stream, 1, x, M, K,
                          ldx, q, ldq, scale);
    }
    // Smallest power-of-two group (>= 8 threads) that covers the row with <= 4 vectors each.
    int tpr = 8;
    while (tpr * 4 < nvec) tpr *= 2;
    const bool two = nvec <= tpr * 2;
#define FP8DIT_Q_CASE(T)                                                                        \
    case T:                                                                                     \
        return two ? launch_regs<T, 2, FMT>(x, M, K, ldx, q, ldq, scale, stream, dev)           \
                   : launch_regs<T, 4, FMT>(x, M, K, ldx, q, ldq, scale, stream, dev);
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

// Exhaustive comparison of the quantisers' code path with IEEE division:
// thread i takes amax = bf16 pattern (i + 1) and, for every bf16 magnitude
// m <= amax, encodes the pair (+m, -m) exactly as the kernels do
// (codes2 + signs4) and as cvt(x / S) with the IEEE division, counting
// differing codes.
template <int FMT>
__device__ unsigned long long selftest_amax(uint32_t amax_bits) {
    const ScaleCtx c = scale_ctx<FMT>(bf16_bits_to_float(amax_bits));
    const Quot2 q = quot2_of(c);
    unsigned long long bad = 0;
    for (uint32_t mag = 0; mag <= amax_bits; ++mag) {
        const uint32_t w = mag | ((mag | 0x8000u) << 16);
        const uint32_t got = ((c.fast ? codes2<FMT, true>(w, q) : codes2<FMT, false>(w, q)) | signs4(w, 0u)) & 0xffffu;
        const float2 ref = make_float2(__fdiv_rn(bf16_lo(w), c.s), __fdiv_rn(bf16_hi(w), c.s));
        const uint32_t want = (uint32_t)__nv_cvt_float2_to_fp8x2(ref, __NV_SATFINITE, Fp8Fmt<FMT>::kInterp) & 0xffffu;
        const uint32_t diff = got ^ want;
        bad += ((diff & 0xffu) != 0) + ((diff >> 8) != 0);
    }
    return bad;
}

__global__ void selftest_quotient_kernel(unsigned long long* mismatch) {
    const uint32_t amax_bits = blockIdx.x * blockDim.x + threadIdx.x + 1;
    if (amax_bits > 0x7F7Fu) return;
    const unsigned long long bad4 = selftest_amax<FP8DIT_E4M3FN>(amax_bits);
    const unsigned long long bad5 = selftest_amax<FP8DIT_E5M2>(amax_bits);
    if (bad4) atomicAdd(&mismatch[0], bad4);
    if (bad5) atomicAdd(&mismatch[1], bad5);
}

}  // namespace

cudaError_t launch_quantize_rows(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int fmt, uint8_t* q,
                                 int64_t ldq, float* scale, cudaStream_t stream, const DeviceInfo* dev) {
    if (M == 0) return cudaSuccess;
    return fmt == FP8DIT_E4M3FN ? launch_fmt<FP8DIT_E4M3FN>(x, M, K, ldx, q, ldq, scale, stream, dev)
                                : launch_fmt<FP8DIT_E5M2>(x, M, K, ldx, q, ldq, scale, stream, dev);
}

cudaError_t launch_selftest_quotient(unsigned long long* mismatch, cudaStream_t stream) {
    const int threads = 128;
    const int blocks = (0x7F7F + threads - 1) / threads;
    selftest_quotient_kernel<<<blocks, threads, 0, stream>>>(mismatch);
    return cudaGetLastError();
}

}  // namespace fp8dit
