// FP8 (E4M3 x E4M3) GEMM with the fused per-token x per-channel scale, bias
// and bf16 epilogue, for sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// What it computes ("从 BF16 到 FP8：HunyuanVideo1.5推理优化复盘", section 三.1,
// the "FP8 GEMM -> scale / bias / output dtype" steps, and section 三.2 item 4:
// the full path with bias, scale and output dtype, not a bare GEMM):
//     y[m, n] = bf16_rne( (sum_k A[m,k] W[n,k]) * sa[m] * sw[n] + bias[n] )
// A [M, K] and W [N, K] are both K-major (the "column-major B" of section 三.1,
// fixed at weight preparation, so no transpose ever reaches this kernel).
//
// Structure (one CTA per SM, persistent over output tiles):
//   warp 0      one thread issues TMA loads of A and W k-blocks (128 B wide,
//               128-byte swizzle) into a STAGES-deep shared-memory ring;
//   warp 1      allocates TMEM; one thread issues tcgen05.mma (M=128, N=BN,
//               K=32 per instruction) into a TMEM accumulator and commits
//               each ring slot back to the producer when its MMAs retire;
//   warps 2..5  epilogue: tcgen05.ld 32 columns at a time, scale, bias, bf16,
//               16-byte global stores; then hand the accumulator back.
// Two TMEM accumulators (2 x BN columns) let the epilogue of tile i overlap
// the mainloop of tile i+1. All mbarrier waits are bounded (see
// mbar_wait_bounded): on expiry the CTA raises the device error word, drains
// its in-flight copies and MMAs, frees TMEM and returns.
#include <cuda_bf16.h>

#include "fp8dit_internal.cuh"

namespace fp8dit {
namespace {

template <int BN>
struct Cfg {
    static constexpr int BM = kGemmBlockM;
    static constexpr int BK = kGemmBlockK;
    static constexpr int STAGES = BN == 256 ? 4 : 6;
    static constexpr int A_BYTES = BM * BK;
    static constexpr int B_BYTES = BN * BK;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int ACC = 2;  // TMEM accumulator buffers
    static constexpr uint32_t TMEM_COLS = ACC * BN;
    static constexpr int BAR_BYTES = 256;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES;
    static constexpr int THREADS = 192;
    static_assert(TMEM_COLS == 256 || TMEM_COLS == 512, "TMEM allocation must be a power of two");
    static_assert((2 * STAGES + 2 * ACC + 1) * 8 + 8 <= BAR_BYTES, "barrier area");
};

struct TileCoord {
    int g, tm, tn;
};

__device__ __forceinline__ TileCoord tile_coord(const GemmArgs& a, int t) {
    int g = 0;
#pragma unroll
    for (int i = 1; i < kMaxGroups; ++i)
        if (i < a.G && t >= a.prob[i].tile_start) g = i;
    const int local = t - a.prob[g].tile_start;
    return TileCoord{g, local % a.tiles_m, local / a.tiles_m};
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

template <int BN>
__global__ void __launch_bounds__(Cfg<BN>::THREADS, 1) gemm_e4m3_kernel(const __grid_constant__ GemmArgs args) {
    using C = Cfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + C::STAGES * C::A_BYTES;
    uint64_t* full = reinterpret_cast<uint64_t*>(sB + C::STAGES * C::B_BYTES);
    uint64_t* empty = full + C::STAGES;
    uint64_t* tfull = empty + C::STAGES;
    uint64_t* tempty = tfull + C::ACC;
    uint64_t* drain = tempty + C::ACC;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < C::ACC; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 4);  // one arrival per epilogue warp
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
        tma_prefetch_desc(&args.tmA);
        for (int g = 0; g < args.G; ++g) tma_prefetch_desc(&args.tmB[g]);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            int64_t armed = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < args.num_tiles && ok; t += gridDim.x) {
                const TileCoord tc = tile_coord(args, t);
                for (int kb = 0; kb < args.num_kb; ++kb) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, args.err)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
                    tma_load_2d(sA + stage * C::A_BYTES, &args.tmA, &full[stage], kb * C::BK, tc.tm * C::BM);
                    tma_load_2d(sB + stage * C::B_BYTES, &args.tmB[tc.g], &full[stage], kb * C::BK, tc.tn * BN);
                    ++armed;
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                // Let every copy this thread started land before the CTA exits.
                DevErr drain_err = args.err;
                for (int s = 0; s < C::STAGES; ++s) {
                    if (armed <= s) break;
                    const int64_t last = s + (int64_t)C::STAGES * ((armed - 1 - s) / C::STAGES);
                    mbar_wait_bounded(&full[s], (uint32_t)((last / C::STAGES) & 1), nullptr, drain_err);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_e4m3_f32(C::BM, BN);
            uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < args.num_tiles && ok; t += gridDim.x) {
                if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag, args.err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * BN;
                for (int kb = 0; kb < args.num_kb; ++kb) {
                    if (!mbar_wait_bounded(&full[stage], phase, abort_flag, args.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sA + stage * C::A_BYTES);
                    const uint32_t b0 = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
                    for (int j = 0; j < C::BK / 32; ++j)
                        mma_f8f6f4(d_tmem, umma_desc_kmajor_sw128(a0 + 32 * j), umma_desc_kmajor_sw128(b0 + 32 * j),
                                   idesc, (kb | j) != 0);
                    mma_commit(&empty[stage]);  // slot free once these MMAs have read it
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit(&tfull[acc]);  // accumulator ready for the epilogue
                if (++acc == C::ACC) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            // Every MMA this thread issued has completed once `drain` fires.
            mma_commit(drain);
            mbar_wait_bounded(drain, 0, nullptr, args.err);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue warps
        const int quarter = warp & 3;  // TMEM lanes [32*quarter, 32*quarter+32)
        uint32_t acc = 0, acc_phase = 0;
        for (int t = blockIdx.x; t < args.num_tiles; t += gridDim.x) {
            const TileCoord tc = tile_coord(args, t);
            // Every lane waits; the warp then agrees (and reconverges) before
            // the warp-collective TMEM loads.
            const bool ready = mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, args.err);
            if (!__all_sync(0xffffffffu, ready)) break;
            tc_fence_after();
            const GemmProblem& P = args.prob[tc.g];
            const int row = tc.tm * C::BM + quarter * 32 + lane;
            const bool row_ok = row < args.M;
            const float sa = row_ok ? __ldg(args.sa + row) : 0.0f;
            uint16_t* yrow = P.y + (int64_t)(row_ok ? row : 0) * P.N;
            const uint32_t t_addr = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * BN;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                const int n0 = tc.tn * BN + c * 32;
                if (n0 >= P.N) break;  // warp-uniform
                uint32_t r[32];
                tmem_ld_32x32b_x32(t_addr + c * 32, r);
                tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int n = n0 + q * 8;
                    if (n < P.N) {
                        const float4 w0 = __ldg(reinterpret_cast<const float4*>(P.sw + n));
                        const float4 w1 = __ldg(reinterpret_cast<const float4*>(P.sw + n + 4));
                        uint4 bb = make_uint4(0, 0, 0, 0);
                        if (P.bias != nullptr) bb = __ldg(reinterpret_cast<const uint4*>(P.bias + n));
                        const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                        const uint32_t bw[4] = {bb.x, bb.y, bb.z, bb.w};
                        float o[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float b = __uint_as_float(e & 1 ? (bw[e >> 1] & 0xffff0000u) : (bw[e >> 1] << 16));
                            o[e] = fmaf(__uint_as_float(r[q * 8 + e]) * sa, wv[e], b);
                        }
                        uint4 packed;
                        packed.x = pack_bf16x2(o[0], o[1]);
                        packed.y = pack_bf16x2(o[2], o[3]);
                        packed.z = pack_bf16x2(o[4], o[5]);
                        packed.w = pack_bf16x2(o[6], o[7]);
                        if (row_ok) *reinterpret_cast<uint4*>(yrow + n) = packed;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
            if (++acc == C::ACC) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

template <int BN>
cudaError_t launch_bn(const GemmArgs& args, int ctas, cudaStream_t stream) {
    using C = Cfg<BN>;
    static bool attr_done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 64 && !attr_done[dev]) {
        e = cudaFuncSetAttribute(gemm_e4m3_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_done[dev] = true;
    }
    gemm_e4m3_kernel<BN><<<ctas, C::THREADS, C::SMEM_BYTES, stream>>>(args);
    return cudaGetLastError();
}

}  // namespace

int gemm_block_n(int cfg) { return cfg == kCfg128x256 ? 256 : 128; }

int gemm_ctas_for(int cfg, int num_tiles, const DeviceInfo* dev) {
    (void)cfg;
    return num_tiles < dev->num_sms ? num_tiles : dev->num_sms;
}

cudaError_t launch_gemm(int cfg, const GemmArgs& args, int ctas, cudaStream_t stream) {
    switch (cfg) {
        case kCfg128x256:
            return launch_bn<256>(args, ctas, stream);
        case kCfg128x128:
            return launch_bn<128>(args, ctas, stream);
        default:
            return cudaErrorInvalidValue;
    }
}

}  // namespace fp8dit
