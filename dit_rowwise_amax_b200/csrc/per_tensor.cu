// Per-tensor amax conversion of a weight set to FP8 ("Quantize Model to FP8
// Format": every tensor of model_state_dict scaled and cast to float8_e4m3fn
// or float8_e5m2). Per tensor: amax = max |W|, S = amax / fmax (IEEE fp32
// division; S = 1 for an all-zero tensor), q = RNE-saturating FP8 of W / S.
//
// Design: a tensor's quantisation needs the amax of the whole tensor, so each
// tensor is read twice. One launch walks a work queue of 32 Ki-element chunks
// ordered so that stage j holds the amax chunks of tensor j followed by the
// quantise chunks of tensor j-1: the second read of a tensor comes one tensor
// later, while it is still in L2 (126 MB; the largest tensor is 32 MB).
// Blocks claim chunks with one atomic per chunk. An amax chunk folds its max
// into the tensor's amax word and then counts itself done (release); a
// quantise chunk waits (acquire, bounded) until all amax chunks of its tensor
// are done. Chunks are claimed in queue order by running blocks, and amax
// chunks never wait, so every wait is on work already held by a running
// block: the launch cannot deadlock whatever the grid size.
#include <cuda_fp16.h>

#include <algorithm>

#include "fp8_codec.cuh"

namespace fp8dit {
namespace {

constexpr int kThreads = 256;
constexpr int kBatch = 192;              // tensors per launch (descriptors travel as kernel parameters)
constexpr int64_t kChunk = 32768;        // elements per work item

struct PerTensorArgs {
    PerTensorDevDesc d[kBatch];
    int64_t chunks[kBatch];
    int64_t stage_start[kBatch + 2];  // first queue index of stage j, j = 0..n; [n+1] = total
    int32_t n;
    unsigned long long* queue;
    uint32_t* amax_bits;  // [kBatch]
    uint32_t* done;       // [kBatch]
    DevErr err;
};

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void red_add_release_gpu(uint32_t* p, uint32_t v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// ---- source element types. A 16-byte vector holds 8 bf16 / fp16 values or
// 4 fp32 values; the amax is kept as the bit pattern of |x| in the source
// type (for non-negative values bit-pattern order is value order).
template <int SRC>
struct Src {
    static constexpr int kEpv = SRC == FP8DIT_SRC_F32 ? 4 : 8;  // elements per 16-byte vector
};

template <int SRC>
__device__ __forceinline__ float abs_bits_to_float(uint32_t bits) {
    if constexpr (SRC == FP8DIT_SRC_BF16) return bf16_bits_to_float(bits);
    else if constexpr (SRC == FP8DIT_SRC_F16) return __half2float(__ushort_as_half((unsigned short)bits));
    else return __uint_as_float(bits);
}

// |x| bits of element e (tails).
template <int SRC>
__device__ __forceinline__ uint32_t abs_bits1(const void* src, int e) {
    if constexpr (SRC == FP8DIT_SRC_F32) return __float_as_uint(static_cast<const float*>(src)[e]) & 0x7fffffffu;
    else return (uint32_t)static_cast<const uint16_t*>(src)[e] & 0x7fffu;
}

// Running max of |x| over a vector: packed pairs for the 16-bit types (folded
// by the caller), one word for fp32.
template <int SRC>
__device__ __forceinline__ uint32_t absmax_vec(const uint4& v, uint32_t acc) {
    if constexpr (SRC == FP8DIT_SRC_BF16) {
        return absmax8(v, acc);
    } else if constexpr (SRC == FP8DIT_SRC_F16) {
        acc = __vmaxu2(acc, v.x & 0x7fff7fffu);
        acc = __vmaxu2(acc, v.y & 0x7fff7fffu);
        acc = __vmaxu2(acc, v.z & 0x7fff7fffu);
        return __vmaxu2(acc, v.w & 0x7fff7fffu);
    } else {
        acc = max(acc, v.x & 0x7fffffffu);
        acc = max(acc, v.y & 0x7fffffffu);
        acc = max(acc, v.z & 0x7fffffffu);
        return max(acc, v.w & 0x7fffffffu);
    }
}

// FP8 codes of two fp32 values divided by s (IEEE division), low element first.
template <int FMT>
__device__ __forceinline__ uint32_t codes2_div(float lo, float hi, float s) {
    return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(lo, s), __fdiv_rn(hi, s)), __NV_SATFINITE,
                                              Fp8Fmt<FMT>::kInterp);
}

// fp16 / fp32 sources: one vector -> its codes (8 bytes for fp16, 4 for fp32,
// as the low bytes of a uint2). Every quotient is the IEEE division x / S (the
// corrected-reciprocal quotient of the bf16 kernels is proven for bf16 inputs
// only); each code takes its sign bit from x.
template <int SRC, int FMT>
__device__ __forceinline__ uint2 quant_vec_div(const uint4& v, float s) {
    if constexpr (SRC == FP8DIT_SRC_F16) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t c[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
            c[k] = codes2_div<FMT>(f.x, f.y, s);
        }
        return make_uint2((c[0] | (c[1] << 16)) | signs4(w[0], w[1]), (c[2] | (c[3] << 16)) | signs4(w[2], w[3]));
    } else {
        const uint32_t c = codes2_div<FMT>(__uint_as_float(v.x), __uint_as_float(v.y), s) |
                           (codes2_div<FMT>(__uint_as_float(v.z), __uint_as_float(v.w), s) << 16);
        const uint32_t signs = ((v.x >> 24) & 0x80u) | ((v.y >> 16) & 0x8000u) | ((v.z >> 8) & 0x800000u) |
                               (v.w & 0x80000000u);
        return make_uint2(c | signs, 0u);
    }
}

// One element -> its code (tails), for any source type.
template <int SRC, int FMT>
__device__ __forceinline__ uint8_t quant1_any(const void* src, int e, const ScaleCtx& c) {
    if constexpr (SRC == FP8DIT_SRC_BF16) {
        return quant1<FMT>(static_cast<const uint16_t*>(src)[e], c);
    } else {
        float x;
        uint32_t sign;
        if constexpr (SRC == FP8DIT_SRC_F16) {
            const uint16_t b = static_cast<const uint16_t*>(src)[e];
            x = __half2float(__ushort_as_half(b));
            sign = (b >> 8) & 0x80u;
        } else {
            x = static_cast<const float*>(src)[e];
            sign = (__float_as_uint(x) >> 24) & 0x80u;
        }
        return (uint8_t)((codes2_div<FMT>(x, 0.0f, c.s) & 0xffu) | sign);
    }
}

// Thread's share of the amax of a chunk of n (<= kChunk) elements starting
// at base, as |x| bits. In-chunk indices are 32-bit.
template <int SRC>
__device__ __forceinline__ uint32_t amax_chunk(const void* base, int n) {
    constexpr int EPV = Src<SRC>::kEpv;
    constexpr int VPT = (int)(kChunk / EPV / kThreads);
    const int nvec = n / EPV;  // whole vectors in this chunk
    const uint4* src = static_cast<const uint4*>(base);
    uint32_t packed = 0;
#pragma unroll 4
    for (int i = 0; i < VPT; ++i) {
        const int vi = i * kThreads + (int)threadIdx.x;
        if (vi < nvec) packed = absmax_vec<SRC>(__ldg(src + vi), packed);
    }
    uint32_t m = SRC == FP8DIT_SRC_F32 ? packed : fold_halves(packed);
    for (int e = nvec * EPV + (int)threadIdx.x; e < n; e += kThreads) m = max(m, abs_bits1<SRC>(base, e));
    return m;
}

// Codes of a chunk of n (<= kChunk) elements from base into dst, with scale
// context c.
template <int SRC, int FMT>
__device__ __forceinline__ void quant_chunk(const void* base, uint8_t* dst, int n, const ScaleCtx& c) {
    constexpr int EPV = Src<SRC>::kEpv;
    constexpr int VPT = (int)(kChunk / EPV / kThreads);
    const int nvec = n / EPV;
    const uint4* src = static_cast<const uint4*>(base);
    if constexpr (SRC == FP8DIT_SRC_BF16) {
        const Quot2 q2 = quot2_of(c);
        if (c.fast) {
#pragma unroll 4
            for (int i = 0; i < VPT; ++i) {
                const int vi = i * kThreads + (int)threadIdx.x;
                if (vi < nvec) __stcs(reinterpret_cast<uint2*>(dst) + vi, quant8<FMT, true>(__ldcs(src + vi), q2));
            }
        } else {
#pragma unroll 4
            for (int i = 0; i < VPT; ++i) {
                const int vi = i * kThreads + (int)threadIdx.x;
                if (vi < nvec) __stcs(reinterpret_cast<uint2*>(dst) + vi, quant8<FMT, false>(__ldcs(src + vi), q2));
            }
        }
    } else if constexpr (SRC == FP8DIT_SRC_F16) {
#pragma unroll 4
        for (int i = 0; i < VPT; ++i) {
            const int vi = i * kThreads + (int)threadIdx.x;
            if (vi < nvec) __stcs(reinterpret_cast<uint2*>(dst) + vi, quant_vec_div<SRC, FMT>(__ldcs(src + vi), c.s));
        }
    } else {
#pragma unroll 4
        for (int i = 0; i < VPT; ++i) {
            const int vi = i * kThreads + (int)threadIdx.x;
            if (vi < nvec) __stcs(reinterpret_cast<uint32_t*>(dst) + vi, quant_vec_div<SRC, FMT>(__ldcs(src + vi), c.s).x);
        }
    }
    for (int e = nvec * EPV + (int)threadIdx.x; e < n; e += kThreads) dst[e] = quant1_any<SRC, FMT>(base, e, c);
}

template <int FMT>
__global__ void __launch_bounds__(kThreads) per_tensor_kernel(const __grid_constant__ PerTensorArgs a) {
    __shared__ unsigned long long s_item;
    __shared__ uint32_t s_red[kThreads / 32];
    __shared__ float s_amax;
    __shared__ int s_ok;
    const unsigned long long total = (unsigned long long)a.stage_start[a.n + 1];

    while (true) {
        if (threadIdx.x == 0) s_item = atomicAdd(a.queue, 1ull);
        __syncthreads();
        const unsigned long long item = s_item;
        if (item >= total) break;

        // Stage j: largest j with stage_start[j] <= item.
        int lo = 0, hi = a.n;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if ((unsigned long long)a.stage_start[mid] <= item) lo = mid;
            else hi = mid - 1;
        }
        const int j = lo;
        int64_t off = (int64_t)(item - (unsigned long long)a.stage_start[j]);
        const int64_t amax_chunks_here = (j < a.n) ? a.chunks[j] : 0;
        const bool is_amax = off < amax_chunks_here;
        const int t = is_amax ? j : j - 1;
        const int64_t chunk = is_amax ? off : off - amax_chunks_here;
        // Per item only the chunk's pointers, its length and the dtype stay
        // live through the loops (32-bit in-chunk indices).
        const PerTensorDevDesc& d = a.d[t];
        const int src_dtype = d.src_dtype;  // uniform across the block (one tensor per item)
        const int64_t begin = chunk * kChunk;
        const int n = (int)min((int64_t)kChunk, d.numel - begin);
        const void* base = static_cast<const uint8_t*>(d.src) + begin * (src_dtype == FP8DIT_SRC_F32 ? 4 : 2);

        if (is_amax) {
            uint32_t m = src_dtype == FP8DIT_SRC_F32   ? amax_chunk<FP8DIT_SRC_F32>(base, n)
                         : src_dtype == FP8DIT_SRC_F16 ? amax_chunk<FP8DIT_SRC_F16>(base, n)
                                                       : amax_chunk<FP8DIT_SRC_BF16>(base, n);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
            if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = m;
            __syncthreads();
            if (threadIdx.x == 0) {
                uint32_t mm = s_red[0];
#pragma unroll
                for (int w = 1; w < kThreads / 32; ++w) mm = max(mm, s_red[w]);
                atomicMax(&a.amax_bits[t], mm);
                red_add_release_gpu(&a.done[t], 1u);  // orders the atomicMax before the count
            }
        } else {
            if (threadIdx.x == 0) {
                const uint32_t need = (uint32_t)a.chunks[t];
                bool ok = ld_acquire_gpu(&a.done[t]) == need;
                if (!ok) {
                    const unsigned long long t0 = globaltimer_ns();
                    while (true) {
                        __nanosleep(256);
                        if (ld_acquire_gpu(&a.done[t]) == need) {
                            ok = true;
                            break;
                        }
                        if (globaltimer_ns() - t0 > a.err.limit_ns) {
                            atomicOr(a.err.word, kDevErrTimeout);
                            break;
                        }
                    }
                }
                const uint32_t bits = ld_acquire_gpu(&a.amax_bits[t]);
                const float amax = src_dtype == FP8DIT_SRC_F32   ? abs_bits_to_float<FP8DIT_SRC_F32>(bits)
                                   : src_dtype == FP8DIT_SRC_F16 ? abs_bits_to_float<FP8DIT_SRC_F16>(bits)
                                                                 : abs_bits_to_float<FP8DIT_SRC_BF16>(bits);
                s_amax = amax;
                s_ok = ok;
                if (ok && chunk == 0) *d.scale = scale_ctx<FMT>(amax).s;
            }
            __syncthreads();
            if (s_ok) {
                const ScaleCtx c = scale_ctx<FMT>(s_amax);
                uint8_t* dst = d.dst + begin;
                if (src_dtype == FP8DIT_SRC_F32) quant_chunk<FP8DIT_SRC_F32, FMT>(base, dst, n, c);
                else if (src_dtype == FP8DIT_SRC_F16) quant_chunk<FP8DIT_SRC_F16, FMT>(base, dst, n, c);
                else quant_chunk<FP8DIT_SRC_BF16, FMT>(base, dst, n, c);
            }
        }
        __syncthreads();  // s_item / s_red / s_amax are rewritten next iteration
    }
}

}  // namespace

size_t per_tensor_workspace_bytes(int32_t n) {
    (void)n;
    // queue counter, then amax words and done counters for one batch.
    return 256 + 2 * sizeof(uint32_t) * kBatch;
}

cudaError_t launch_per_tensor(const fp8dit_tensor_desc* host_descs, int32_t n, int fmt, void* ws,
                              cudaStream_t stream, const DeviceInfo* dev, DevErr err) {
    uint8_t* w = static_cast<uint8_t*>(ws);
    PerTensorArgs args;
    args.queue = reinterpret_cast<unsigned long long*>(w);
    args.amax_bits = reinterpret_cast<uint32_t*>(w + 256);
    args.done = args.amax_bits + kBatch;
    args.err = err;
    for (int32_t base = 0; base < n; base += kBatch) {
        const int32_t nb = std::min<int32_t>(kBatch, n - base);
        args.n = nb;
        int64_t total_chunks = 0;
        for (int32_t i = 0; i < nb; ++i) {
            const fp8dit_tensor_desc& h = host_descs[base + i];
            args.d[i] = PerTensorDevDesc{h.src, h.numel, h.dst, h.scale, h.src_dtype};
            args.chunks[i] = (h.numel + kChunk - 1) / kChunk;
            total_chunks += args.chunks[i];
        }
        if (total_chunks == 0) continue;
        int64_t pos = 0;
        for (int32_t j = 0; j <= nb; ++j) {
            args.stage_start[j] = pos;
            if (j < nb) pos += args.chunks[j];
            if (j >= 1) pos += args.chunks[j - 1];
        }
        args.stage_start[nb + 1] = pos;
        cudaError_t e = cudaMemsetAsync(ws, 0, per_tensor_workspace_bytes(nb), stream);
        if (e != cudaSuccess) return e;
        // A persistent grid: as many blocks as are resident at once (blocks
        // beyond that would only start once the queue is drained).
        void (*kernel)(PerTensorArgs) =
            fmt == FP8DIT_E4M3FN ? per_tensor_kernel<FP8DIT_E4M3FN> : per_tensor_kernel<FP8DIT_E5M2>;
        static int per_sm[2] = {0, 0};  // resident blocks per SM, per format (same on every sm_100a device)
        int& resident = per_sm[fmt == FP8DIT_E4M3FN ? 0 : 1];
        if (resident == 0) {
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&resident, kernel, kThreads, 0);
            if (e != cudaSuccess) return e;
            if (resident < 1) resident = 1;
        }
        const int64_t grid = std::min<int64_t>((int64_t)dev->num_sms * resident, total_chunks * 2);
        kernel<<<(unsigned)grid, kThreads, 0, stream>>>(args);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace fp8dit
