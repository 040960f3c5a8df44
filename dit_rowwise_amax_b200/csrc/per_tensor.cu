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
#include <algorithm>

#include "fp8_codec.cuh"

namespace fp8dit {
namespace {

constexpr int kThreads = 256;
constexpr int kBatch = 192;              // tensors per launch (descriptors travel as kernel parameters)
constexpr int64_t kChunk = 32768;        // elements per work item
constexpr int kVecPerThread = kChunk / 8 / kThreads;  // 16 vectors of 8 bf16

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
        const PerTensorDevDesc d = a.d[t];
        const int64_t begin = chunk * kChunk;
        const int64_t end = min(d.numel, begin + kChunk);
        const int64_t nvec = (end - begin) >> 3;  // whole 8-element vectors in this chunk
        const uint4* src = reinterpret_cast<const uint4*>(d.src + begin);

        if (is_amax) {
            uint32_t packed = 0;
#pragma unroll 4
            for (int i = 0; i < kVecPerThread; ++i) {
                const int64_t vi = (int64_t)i * kThreads + threadIdx.x;
                if (vi < nvec) {
                    packed = absmax8(__ldg(src + vi), packed);
                }
            }
            for (int64_t e = begin + nvec * 8 + threadIdx.x; e < end; e += kThreads)
                packed = absmax2((uint32_t)d.src[e], packed);
            uint32_t m = fold_halves(packed);
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
                const float amax = bf16_bits_to_float(ld_acquire_gpu(&a.amax_bits[t]));
                s_amax = amax;
                s_ok = ok;
                if (ok && chunk == 0) *d.scale = scale_ctx<FMT>(amax).s;
            }
            __syncthreads();
            if (s_ok) {
                const ScaleCtx c = scale_ctx<FMT>(s_amax);
                const Quot2 q2 = quot2_of(c);
                uint8_t* dst = d.dst + begin;
                if (c.fast) {
#pragma unroll 4
                    for (int i = 0; i < kVecPerThread; ++i) {
                        const int64_t vi = (int64_t)i * kThreads + threadIdx.x;
                        if (vi < nvec) __stcs(reinterpret_cast<uint2*>(dst) + vi, quant8<FMT, true>(__ldcs(src + vi), q2));
                    }
                } else {
#pragma unroll 4
                    for (int i = 0; i < kVecPerThread; ++i) {
                        const int64_t vi = (int64_t)i * kThreads + threadIdx.x;
                        if (vi < nvec) __stcs(reinterpret_cast<uint2*>(dst) + vi, quant8<FMT, false>(__ldcs(src + vi), q2));
                    }
                }
                for (int64_t e = begin + nvec * 8 + threadIdx.x; e < end; e += kThreads)
                    d.dst[e] = quant1<FMT>(d.src[e], c);
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
            args.d[i] = PerTensorDevDesc{h.src, h.numel, h.dst, h.scale};
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
        const int64_t grid = std::min<int64_t>((int64_t)dev->num_sms * 8, total_chunks * 2);
        if (fmt == FP8DIT_E4M3FN)
            per_tensor_kernel<FP8DIT_E4M3FN><<<(unsigned)grid, kThreads, 0, stream>>>(args);
        else
            per_tensor_kernel<FP8DIT_E5M2><<<(unsigned)grid, kThreads, 0, stream>>>(args);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace fp8dit
