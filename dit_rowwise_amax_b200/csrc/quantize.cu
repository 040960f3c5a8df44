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
//
// Producer fusion ("从 BF16 到 FP8", section 三.5): with ACT != 0 the kernels
// first replace each loaded element by bf16(act(x)) — GELU (erf or tanh form)
// or SiLU — optionally store that bf16 tensor, and quantise it. A bf16 input
// has only 65536 values, so bf16(act(x)) is evaluated once per device for
// every bf16 pattern into a 128 KB table (act_table_kernel) and the
// quantisers read the table: one cached load per element. Since the table is
// built once, each entry is evaluated in double (CUDA's double erfc / exp, in
// forms that do not cancel for negative x, every other operation an
// explicitly rounded IEEE double operation) and rounded once to bf16, ties to
// even: the correctly rounded activation except where the true value lies
// within a few double ulps of a bf16 rounding boundary.
#include <algorithm>
#include <mutex>

#include "fp8_codec.cuh"

namespace fp8dit {
namespace {

constexpr int kThreads = 256;

// The activation in double. Every product, sum and quotient is an explicitly
// rounded IEEE double operation (no contraction into FMAs), so the only
// inexact steps besides them are CUDA's double erfc and exp:
//   GELU, erf form    (x / 2) erfc(-x / sqrt 2)                 = x Phi(x)
//   GELU, tanh form   x / (1 + exp(-2 sqrt(2/pi) (x + 0.044715 x^3)))
//   SiLU              x / (1 + exp(-x))
// The right-hand forms do not cancel for negative x (1 + erf and 1 + tanh
// would). exp overflowing to +inf gives x / inf = -0 for very negative x.
template <int ACT>
__device__ double act_d(double x) {
    if constexpr (ACT == FP8DIT_ACT_GELU_ERF) {
        return __dmul_rn(__dmul_rn(0.5, x), erfc(__ddiv_rn(-x, __dsqrt_rn(2.0))));
    } else if constexpr (ACT == FP8DIT_ACT_GELU_TANH) {
        const double c = __dmul_rn(-2.0, __dsqrt_rn(__ddiv_rn(2.0, 3.14159265358979323846)));
        const double cube = __dmul_rn(__dmul_rn(__dmul_rn(0.044715, x), x), x);
        return __ddiv_rn(x, __dadd_rn(1.0, exp(__dmul_rn(c, __dadd_rn(x, cube)))));
    } else if constexpr (ACT == FP8DIT_ACT_SILU) {
        return __ddiv_rn(x, __dadd_rn(1.0, exp(-x)));
    } else {
        return x;
    }
}

// Nearest bf16 to a double, ties to even, in one rounding: truncate to fp32
// and set the lowest bit when that dropped anything (round to odd; fp32 keeps
// 16 more significand bits than bf16, subnormals included), then round that
// fp32 to bf16 to nearest even. Rounding to odd with at least two extra bits
// followed by round-to-nearest equals one round-to-nearest (Boldo and
// Melquiond, "Emulation of FMA and correctly rounded sums: proved algorithms
// using rounding to odd", IEEE Trans. Computers 57(4), 2008).
__device__ __forceinline__ uint16_t bf16_rne_of_double(double v) {
    const float f = __double2float_rz(v);
    uint32_t u = __float_as_uint(f);
    if ((double)f != v) u |= 1u;
    const __nv_bfloat16 r = __float2bfloat16_rn(__uint_as_float(u));
    return *reinterpret_cast<const uint16_t*>(&r);
}

// bf16(act(x)) for every bf16 pattern x, one table per activation.
__device__ uint16_t g_act_table[3][65536];

template <int ACT>
__global__ void act_table_kernel() {
    const uint32_t b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= 65536u) return;
    g_act_table[ACT - 1][b] = bf16_rne_of_double(act_d<ACT>((double)__uint_as_float(b << 16)));
}

// bf16(act(x)) for the eight bf16 of a 16-byte vector.
template <int ACT>
__device__ __forceinline__ uint4 act8(const uint4& v) {
    if constexpr (ACT == 0) {
        return v;
    } else {
        const uint16_t* tbl = g_act_table[ACT - 1];
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k)
            w[k] = (uint32_t)__ldg(tbl + (w[k] & 0xffffu)) | ((uint32_t)__ldg(tbl + (w[k] >> 16)) << 16);
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
}

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
template <int TPR, int VPT, int FMT, int ACT>
__global__ void __launch_bounds__(kThreads) quantize_rows_regs(const uint16_t* __restrict__ x, int64_t M,
                                                                 int32_t K, int64_t ldx, uint8_t* __restrict__ q,
                                                                 int64_t ldq, float* __restrict__ scale, int64_t groups,
                                                                 uint16_t* __restrict__ gout, int64_t ldg) {
    constexpr int RPB = kThreads / TPR;
    constexpr int WPR = TPR / 32;  // warps per row (when TPR >= 32)
    __shared__ uint32_t red[2][kThreads / 32];
    const int t = threadIdx.x % TPR;
    const int r = threadIdx.x / TPR;
    const int nvec = K >> 3;

    uint4 cur[VPT], nxt[VPT];
    int64_t g = blockIdx.x;
    // Ask L2 for this block's first rows while the previous kernel in the
    // stream is still finishing: a prefetch only warms L2, which every write
    // of that kernel reaches too, so the loads after pdl_wait() still see its
    // results. Each group is at most 256 threads x VPT x 16 bytes = 16 KB.
    if (threadIdx.x == 0 && g < groups) {
        const int64_t r0 = g * RPB;
        const int64_t nr = M - r0 < RPB ? M - r0 : RPB;
        if (ldx == K) {
            prefetch_l2_bulk(x + r0 * ldx, (uint32_t)(nr * K * 2));
        } else {
            for (int64_t rr = 0; rr < nr; ++rr) prefetch_l2_bulk(x + (r0 + rr) * ldx, (uint32_t)K * 2u);
        }
    }
    pdl_wait();  // x may be the previous kernel's output; q and scale its input
    pdl_trigger();
    load_group<TPR, VPT>(x, M, nvec, ldx, g, cur);
    for (int it = 0; g < groups; g += gridDim.x, ++it) {
        const int64_t gn = g + gridDim.x;
        if (gn < groups) load_group<TPR, VPT>(x, M, nvec, ldx, gn, nxt);
        if constexpr (ACT != 0) {
#pragma unroll
            for (int i = 0; i < VPT; ++i) cur[i] = act8<ACT>(cur[i]);
            const int64_t row = g * RPB + r;
            if (gout != nullptr && row < M) {
                uint4* gr = reinterpret_cast<uint4*>(gout + row * ldg);
#pragma unroll
                for (int i = 0; i < VPT; ++i) {
                    const int vi = i * TPR + t;
                    if (vi < nvec) gr[vi] = cur[i];
                }
            }
        }

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
        }
        if (row < M && t == 0) scale[row] = c.s;
#pragma unroll
        for (int i = 0; i < VPT; ++i) cur[i] = nxt[i];
    }
}

// One block per row (grid-strided): amax pass, then a quantise pass that
// re-reads the row (from L2). For rows beyond the register-resident kernel.
template <int FMT, int ACT>
__global__ void __launch_bounds__(kThreads) quantize_rows_two_pass(const uint16_t* __restrict__ x, int64_t M,
                                                                     int64_t K, int64_t ldx,
                                                                     uint8_t* __restrict__ q, int64_t ldq,
                                                                     float* __restrict__ scale,
                                                                     uint16_t* __restrict__ gout, int64_t ldg) {
    __shared__ uint32_t red[kThreads / 32];
    const int64_t nvec = K >> 3;
    pdl_wait();
    pdl_trigger();
    for (int64_t row = blockIdx.x; row < M; row += gridDim.x) {
        const uint4* xr = reinterpret_cast<const uint4*>(x + row * ldx);
        uint32_t packed = 0;
        for (int64_t vi = threadIdx.x; vi < nvec; vi += kThreads)
            packed = absmax8(act8<ACT>(__ldg(xr + vi)), packed);
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
        if (threadIdx.x == 0) scale[row] = c.s;
        const Quot2 q2 = quot2_of(c);
        uint8_t* qr = q + row * ldq;
        uint4* gr = gout != nullptr ? reinterpret_cast<uint4*>(gout + row * ldg) : nullptr;
        for (int64_t vi = threadIdx.x; vi < nvec; vi += kThreads) {
            const uint4 v = act8<ACT>(__ldcs(xr + vi));
            if (ACT != 0 && gr != nullptr) gr[vi] = v;
            *reinterpret_cast<uint2*>(qr + vi * 8) = c.fast ? quant8<FMT, true>(v, q2) : quant8<FMT, false>(v, q2);
        }
    }
}

struct RowsArgs {
    const uint16_t* x;
    int64_t M, K, ldx;
    uint8_t* q;
    int64_t ldq;
    float* scale;
    uint16_t* g;
    int64_t ldg;
};

template <int TPR, int VPT, int FMT, int ACT>
cudaError_t launch_regs(const RowsArgs& a, cudaStream_t stream, const DeviceInfo* dev) {
    constexpr int RPB = kThreads / TPR;
    static int per_sm = 0;  // resident blocks per SM (same on every sm_100a device)
    if (per_sm == 0) {
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &per_sm, quantize_rows_regs<TPR, VPT, FMT, ACT>, kThreads, 0);
        if (e != cudaSuccess) return e;
        if (per_sm < 1) per_sm = 1;
    }
    const int64_t groups = (a.M + RPB - 1) / RPB;
    const int64_t grid = std::min<int64_t>(groups, (int64_t)dev->num_sms * per_sm);
    return launch_pdl(quantize_rows_regs<TPR, VPT, FMT, ACT>, dim3((unsigned)grid), dim3(kThreads), 0, stream, 1,
                      a.x, a.M, (int32_t)a.K, a.ldx, a.q, a.ldq, a.scale, groups, a.g, a.ldg);
}

template <int FMT, int ACT>
cudaError_t launch_fmt(const RowsArgs& a, cudaStream_t stream, const DeviceInfo* dev) {
    const int64_t nvec = a.K / 8;
    if (nvec > 1024) {
        const int64_t grid = std::min<int64_t>(a.M, (int64_t)dev->num_sms * 8);
        return launch_pdl(quantize_rows_two_pass<FMT, ACT>, dim3((unsigned)grid), dim3(kThreads), 0, stream, 1, a.x,
                          a.M, a.K, a.ldx, a.q, a.ldq, a.scale, a.g, a.ldg);
    }
    // Smallest power-of-two group (>= 8 threads) that covers the row with <= 4 vectors each.
    int tpr = 8;
    while (tpr * 4 < nvec) tpr *= 2;
    const bool two = nvec <= tpr * 2;
#define FP8DIT_Q_CASE(T)                                                                        \
    case T:                                                                                     \
        return two ? launch_regs<T, 2, FMT, ACT>(a, stream, dev) : launch_regs<T, 4, FMT, ACT>(a, stream, dev);
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
    const RowsArgs a{x, M, K, ldx, q, ldq, scale, nullptr, 0};
    return fmt == FP8DIT_E4M3FN ? launch_fmt<FP8DIT_E4M3FN, 0>(a, stream, dev)
                                : launch_fmt<FP8DIT_E5M2, 0>(a, stream, dev);
}

// Builds the activation tables on the current device once (on `stream`, which
// is then synchronised, so later calls on any stream see the tables).
static cudaError_t ensure_act_tables(cudaStream_t stream) {
    static std::mutex mu;
    static bool ready[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (ready[dev]) return cudaSuccess;
    act_table_kernel<FP8DIT_ACT_GELU_ERF><<<256, 256, 0, stream>>>();
    act_table_kernel<FP8DIT_ACT_GELU_TANH><<<256, 256, 0, stream>>>();
    act_table_kernel<FP8DIT_ACT_SILU><<<256, 256, 0, stream>>>();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = cudaStreamSynchronize(stream)) != cudaSuccess) return e;
    ready[dev] = true;
    return cudaSuccess;
}

cudaError_t launch_act_quantize_rows(const uint16_t* h, int64_t M, int64_t K, int64_t ldh, int act, uint8_t* q,
                                     int64_t ldq, float* scale, uint16_t* g, int64_t ldg, cudaStream_t stream,
                                     const DeviceInfo* dev) {
    if (M == 0) return cudaSuccess;
    cudaError_t e = ensure_act_tables(stream);
    if (e != cudaSuccess) return e;
    const RowsArgs a{h, M, K, ldh, q, ldq, scale, g, ldg};
    switch (act) {
        case FP8DIT_ACT_GELU_ERF:
            return launch_fmt<FP8DIT_E4M3FN, FP8DIT_ACT_GELU_ERF>(a, stream, dev);
        case FP8DIT_ACT_GELU_TANH:
            return launch_fmt<FP8DIT_E4M3FN, FP8DIT_ACT_GELU_TANH>(a, stream, dev);
        case FP8DIT_ACT_SILU:
            return launch_fmt<FP8DIT_E4M3FN, FP8DIT_ACT_SILU>(a, stream, dev);
        default:
            return cudaErrorInvalidValue;
    }
}

cudaError_t launch_selftest_quotient(unsigned long long* mismatch, cudaStream_t stream) {
    const int threads = 128;
    const int blocks = (0x7F7F + threads - 1) / threads;
    selftest_quotient_kernel<<<blocks, threads, 0, stream>>>(mismatch);
    return cudaGetLastError();
}

}  // namespace fp8dit
