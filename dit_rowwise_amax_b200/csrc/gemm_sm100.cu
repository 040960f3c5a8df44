// FP8 (E4M3 x E4M3) GEMM with the fused per-token x per-channel scale, bias
// and bf16 epilogue, for sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// What it computes ("从 BF16 到 FP8：HunyuanVideo1.5推理优化复盘", section 三.1,
// the steps after the FP8 GEMM: scales, bias, output type; section 三.2 item 4:
// the full path with bias, scale and output dtype, not a bare GEMM):
//     y[m, n] = bf16_rne( (sum_k A[m,k] W[n,k]) * sa[m] * sw[n] + bias[n] )
// A [M, K] and W [N, K] are both K-major (section 三.1's column-major B operand,
// fixed at weight preparation, so no transpose ever reaches this kernel).
//
// Structure (persistent over output tiles, one CTA per SM):
//   warp 0      one thread issues TMA loads of A and W k-blocks (128 B wide,
//               128-byte swizzle) into a STAGES-deep shared-memory ring;
//   warp 1      allocates TMEM; one thread of the pair's leader CTA issues
//               tcgen05.mma (K = 32 per instruction) into a TMEM accumulator
//               and commits each ring slot back to the producers;
//   warps 2..9  epilogue (kOpsFp8; four warps, one per lane quarter, in the
//               converter modes), two warps per TMEM lane quarter, each taking
//               half of the tile's columns: fetch the next tile's sw / bias / sa
//               while this tile is processed, tcgen05.ld 32 accumulator
//               columns at a time, scale, bias, bf16, write a 32 x 32 box
//               into the warp's 64-byte-swizzled staging buffer and
//               TMA-store it.
// Two TMEM accumulators let the epilogue of tile i overlap the mainloop of
// tile i+1.
//
// CG = 2 runs one MMA across a CTA pair (cta_group::2, a 2-CTA cluster): the
// tile is 256 x BN, each CTA loads its 128 rows of A and BN/2 rows of W, the
// leader issues the MMAs, and each CTA's TMEM receives its 128 output rows.
// Per-SM shared-memory traffic per MMA is half that of a 1-CTA tile, which
// lets a 6-deep ring of 32 KB stages cover the L2 latency. No TMA load
// anywhere uses multicast.
//
// Operand modes (OPS): kOpsFp8 is the FP8 linear above. kOpsW8 (FP8
// weight-only: bf16 A x E4M3 W, "longcat-avatar-compare", section 速度总览)
// adds one converter warp per ring stage after the epilogue warps, which turns
// the stage's W codes into bf16 in place in shared memory before releasing the
// stage to the MMA. kOpsQG (the fused linear) first quantises the bf16 A per
// token with every CTA of the launch (phase Q, see qg_quantise), then runs the
// kOpsFp8 GEMM on the codes.
//
// Schedules: data-parallel (tile t on MMA unit t mod units) or, with a
// workspace, stream-K (each unit an equal share of all k-blocks; a tile split
// between two units is finished by one of them after the other has published
// its fp32 partial) or split-K for few tiles and a long K (one CTA per (tile,
// piece of K); every piece stores its fp32 partial and arrives on the tile's
// counter, and the piece that arrives last adds the pieces in order for the
// whole tile), see SegSched.
//
// Every mbarrier wait is bounded (mbar_wait_bounded): on expiry the CTA
// raises the device error word and its own and its peer's abort flags, lets
// in-flight copies and MMAs land, frees TMEM and returns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "fp8_codec.cuh"
#include "fp8dit_internal.cuh"

namespace fp8dit {
namespace {

// Operand modes of the kernel.
//   kOpsFp8: A and W are FP8 codes, both loaded by TMA (the FP8 linear).
//   kOpsW8:  A is bf16; W codes are decoded to bf16 in shared memory (weight-only).
//   kOpsQG:  A is bf16: the launch's CTAs first quantise it per token into the
//            caller's FP8 scratch (rows claimed chunk by chunk, staged in
//            shared memory), then run the kOpsFp8 GEMM on it, each tile
//            starting once its rows are quantised (the fused linear).
enum : int { kOpsFp8 = 0, kOpsW8 = 1, kOpsQG = 2 };

template <int CG, int BN, int OPS>
struct Cfg {
    static constexpr bool W8 = OPS == kOpsW8;
    static constexpr bool QG = OPS == kOpsQG;
    static constexpr bool CONV = W8;        // has converter warps
    static constexpr int BM = 128 * CG;     // rows of one MMA tile
    static constexpr int ROWS = 128;        // rows per CTA (TMEM lanes)
    static constexpr int ROW_BYTES = 128;   // one 128-byte swizzle row per operand row per stage
    static constexpr int KE = W8 ? 64 : 128;  // K elements per stage (bf16 : FP8)
    static constexpr int B_ROWS = BN / CG;  // W rows per CTA per stage
    static constexpr int A_BYTES = ROWS * ROW_BYTES;  // MMA-ready A per stage
    static constexpr int A_STAGE = A_BYTES;
    static constexpr int B_BYTES = B_ROWS * ROW_BYTES;         // MMA-ready B: FP8, or bf16 decoded from FP8
    // W8: the FP8 weight codes as loaded (B_ROWS rows x 64 bytes) land in the
    // upper half of the stage's B buffer and are decoded in place.
    static constexpr int RAW_BYTES = W8 ? B_ROWS * 64 : 0;
    static constexpr int TX_BYTES = A_STAGE + (W8 ? RAW_BYTES : B_BYTES);  // TMA bytes per CTA per stage
    static constexpr int STAGE_SMEM = A_STAGE + B_BYTES;
    static constexpr int STAGES = W8 ? 6 : ((CG == 2) ? (BN == 256 ? 6 : 8) : (BN == 256 ? 4 : BN == 64 ? 8 : 6));
    static constexpr int ACC = 2;
    static constexpr uint32_t TMEM_COLS = ACC * BN;
    static constexpr int EPI_WARPS = CONV ? 4 : 8;   // one or two per TMEM lane quarter
    // Split-K is compiled only into the 128 x 128 single-CTA kernels of the FP8
    // linear and of the weight-only linear.
    static constexpr bool SPLIT_OK = CG == 1 && BN == 128 && (OPS == kOpsFp8 || OPS == kOpsW8);
    static constexpr int HALVES = EPI_WARPS / 4;  // epilogue warps per TMEM lane quarter
    static constexpr int CONV_WARPS = CONV ? STAGES : 0;  // converter warps, one per ring stage
    static constexpr int EPI_COLS = BN / (EPI_WARPS / 4);  // columns per epilogue warp
    static constexpr int BOX = 32;                   // epilogue store box: 32 rows x 32 columns
    static constexpr int STG_BYTES = BOX * BOX * 2;  // 2 KB, 64-byte rows, one per epilogue warp
    static constexpr int STAGING_BYTES = EPI_WARPS * STG_BYTES;
    static constexpr int SWB_FLOATS = 2 * EPI_COLS;  // sw then bias as fp32, one copy per epilogue warp
    static constexpr int SWB_BYTES = EPI_WARPS * SWB_FLOATS * 4;
    static constexpr int BAR_BYTES = 512;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_SMEM + STAGING_BYTES + SWB_BYTES + BAR_BYTES;
    static constexpr int THREADS = 64 + 32 * (EPI_WARPS + CONV_WARPS);
    static_assert(TMEM_COLS == 128 || TMEM_COLS == 256 || TMEM_COLS == 512, "TMEM allocation must be a power of two");
    static_assert((3 * STAGES + 2 * ACC + 2 + 2 * kQgBufs) * 8 + 4 * (6 + kQgBufs) <= BAR_BYTES, "barrier area");
    // Fused linear: kQgBufs chunks of bf16 rows (kQgBufBytes each) are staged
    // in the operand ring before the GEMM uses it.
    static_assert(!QG || kQgBufs * kQgBufBytes <= STAGES * STAGE_SMEM, "quantiser staging");
    // Split-K reduction: one 32-row quarter of every piece's partial is staged
    // in the (then idle) operand ring.
    static_assert(!SPLIT_OK || kSplitMaxPieces * 32 * BN * 4 <= STAGES * STAGE_SMEM, "split-K staging");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static_assert(!W8 || (B_BYTES == 2 * RAW_BYTES && B_ROWS == 128), "in-place decode layout");
};

struct TileCoord {
    int g, tm, tn;
};

// Tile order within a problem: consecutive indices walk along N (every column
// tile of a row block, then the next row block), and unit u takes tiles u,
// u + units, ... So the tiles in flight together cover few row blocks, each
// A k-slice being streamed by many pairs at once while each W slice is read by
// few. Measured against the M-fastest order on B200 (back-to-back launches
// from an idle start): the FFN GEMMs 1.2-1.3 us (2%) faster, the grouped
// Q/K/V projection of hidden_states 5.6% faster, the weight-only linear
// 2.4-3.3% faster.
__device__ __forceinline__ TileCoord tile_coord(const GemmArgs& a, int t) {
    int g = 0;
#pragma unroll
    for (int i = 1; i < kMaxGroups; ++i)
        if (i < a.G && t >= a.prob[i].tile_start) g = i;
    const int local = t - a.prob[g].tile_start;
    return TileCoord{g, local / a.prob[g].tiles_n, local % a.prob[g].tiles_n};
}

// The work of one MMA unit as a sequence of segments (tile t, k-blocks
// [k0, k1)). Data-parallel: whole tiles unit, unit + units, ... Stream-K: the
// unit's equal share [pos, end) of the num_tiles x num_kb k-blocks, cut at
// tile boundaries. With num_tiles >= units a share spans at least one tile,
// so a tile has at most two segments: a head [0, a) that ends its unit's
// share and a tail [a, num_kb) that starts the next unit's share. Split-K:
// piece p of tile t (work item t * split + p, items dealt round-robin) covers
// k-blocks [p * num_kb / split, (p + 1) * num_kb / split).
struct Segment {
    int t, k0, k1, piece;
};
struct SegSched {
    int64_t pos, end;
    int step, num_kb, split;
    bool sk;
};
__device__ __forceinline__ SegSched seg_begin(const GemmArgs& a, int unit, int units, bool split_ok) {
    SegSched s;
    s.sk = a.stream_k != 0;
    s.num_kb = a.num_kb;
    s.split = split_ok && a.split_k > 1 ? a.split_k : 1;
    if (s.split > 1) {
        s.pos = unit;
        s.end = (int64_t)a.num_tiles * s.split;
        s.step = units;
    } else if (s.sk) {
        const int64_t total = (int64_t)a.num_tiles * a.num_kb;
        s.pos = total * unit / units;
        s.end = total * (unit + 1) / units;
        s.step = 0;
    } else {
        s.pos = unit;
        s.end = a.num_tiles;
        s.step = units;
    }
    return s;
}
__device__ __forceinline__ bool seg_next(SegSched& s, Segment& g) {
    if (s.pos >= s.end) return false;
    g.piece = 0;
    if (s.split > 1) {
        g.t = (int)(s.pos / s.split);
        g.piece = (int)(s.pos % s.split);
        g.k0 = (int)((int64_t)g.piece * s.num_kb / s.split);
        g.k1 = (int)((int64_t)(g.piece + 1) * s.num_kb / s.split);
        s.pos += s.step;
    } else if (s.sk) {
        g.t = (int)(s.pos / s.num_kb);
        g.k0 = (int)(s.pos % s.num_kb);
        const int64_t tile_end = (int64_t)(g.t + 1) * s.num_kb;
        const int64_t stop = tile_end < s.end ? tile_end : s.end;
        g.k1 = g.k0 + (int)(stop - s.pos);
        s.pos = stop;
    } else {
        g.t = (int)s.pos;
        g.k0 = 0;
        g.k1 = s.num_kb;
        s.pos += s.step;
    }
    return true;
}

__device__ __forceinline__ uint32_t ld_acquire_gpu_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t atom_acq_rel_gpu_add_u32(uint32_t* p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}
// Wait (acquire, bounded) until *p == want. Gives up when *abort becomes
// non-zero or after err.limit_ns (then raises *abort and the error word).
__device__ __forceinline__ bool wait_count_bounded(const uint32_t* p, uint32_t want, volatile int* abort,
                                                   const DevErr& err) {
    if (ld_acquire_gpu_u32(p) == want) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (true) {
        __nanosleep(64);
        if (ld_acquire_gpu_u32(p) == want) return true;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > err.limit_ns) {
            *abort = 1;
            atomicOr(err.word, kDevErrTimeout);
            return false;
        }
    }
}
__device__ __forceinline__ void red_add_release_gpu_u32(uint32_t* p, uint32_t v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t atom_exch_acq_rel_gpu_u32(uint32_t* p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.exch.b32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

template <int CG, int BN, int OPS>
__global__ void __launch_bounds__(Cfg<CG, BN, OPS>::THREADS, 1)
    gemm_e4m3_kernel(const __grid_constant__ GemmArgs args) {
    using C = Cfg<CG, BN, OPS>;
    constexpr bool W8 = C::W8;
    constexpr bool CONV = C::CONV;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = sA + C::STAGES * C::A_STAGE;
    uint8_t* staging = sB + C::STAGES * C::B_BYTES;
    float* swb = reinterpret_cast<float*>(staging + C::STAGING_BYTES);
    uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(swb) + C::SWB_BYTES);
    uint64_t* empty = full + C::STAGES;
    uint64_t* conv = empty + C::STAGES;  // W8: converted stage ready (arrivals from both CTAs' converters)
    uint64_t* tfull = conv + C::STAGES;
    uint64_t* tempty = tfull + C::ACC;
    uint64_t* drain = tempty + C::ACC;
    uint64_t* redbar = drain + 1;  // split-K: staged partial quarters landed
    uint64_t* qfull = redbar + 1;     // fused linear: a staged chunk of bf16 rows landed
    uint64_t* qempty = qfull + kQgBufs;  // fused linear: a staging buffer is free again
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qempty + kQgBufs);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile uint32_t* split_ticket = reinterpret_cast<volatile uint32_t*>(tmem_slot + 2);  // split-K
    volatile uint32_t* split_fail = reinterpret_cast<volatile uint32_t*>(tmem_slot + 3);    // split-K
    volatile uint32_t* split_ok = reinterpret_cast<volatile uint32_t*>(tmem_slot + 4);      // split-K
    volatile int* qchunk = reinterpret_cast<volatile int*>(tmem_slot + 5);  // fused: chunk in each buffer [kQgBufs]
    volatile uint32_t* qlast = tmem_slot + 5 + kQgBufs;  // fused: this CTA finished last

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = (CG == 2) ? cluster_ctarank() : 0u;
    const bool leader = rank == 0;
    const int unit = (CG == 2) ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;  // MMA unit (pair or CTA)
    const int units = (CG == 2) ? (int)(gridDim.x >> 1) : (int)gridDim.x;

    // Tell the other CTA of the pair to stop waiting (after our own wait expired).
    auto abort_peer = [&]() {
        if (CG == 2) st_shared_cluster_u32(mapa_shared(smem_u32((const void*)abort_flag), rank ^ 1u), 1u);
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&conv[s], CG);  // the stage's converter warp in each CTA (W8)
        }
        for (int a = 0; a < C::ACC; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], C::EPI_WARPS * CG);  // one arrival per epilogue warp of the pair
        }
        mbar_init(drain, 1);
        mbar_init(redbar, 1);
        for (int b = 0; b < kQgBufs; ++b) {
            mbar_init(&qfull[b], 1);
            mbar_init(&qempty[b], 1);
        }
        *abort_flag = 0;
        *split_ticket = 0u;
        *split_fail = 0u;
        *split_ok = 0u;
        fence_mbarrier_init();
        tma_prefetch_desc(&args.tmA);
        for (int g = 0; g < args.G; ++g) {
            tma_prefetch_desc(&args.tmB[g]);
            tma_prefetch_desc(&args.tmY[g]);
        }
    }
    if (warp == 1) {
        if (CG == 2) {
            tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(tmem_slot, C::TMEM_COLS);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (CG == 2) cluster_sync_all();  // peer barriers initialised before any remote signal
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    bool aborted = false;
    // The prologue above touched no global memory; from here on A, W, the
    // scales and y may belong to the previous kernel in the stream.
    pdl_wait();
    pdl_trigger();

    if constexpr (C::QG) {
        // ------------------------------------------------ phase Q (fused linear)
        // Every CTA quantises rows of A until none are left unclaimed. Thread
        // 0 claims chunks of qg_rows rows in row order (kQgClaim chunks per
        // atomic) and bulk-copies chunk i of this CTA into
        // staging buffer i mod 8 in the operand ring. Quantising warp w owns
        // buffer w: for each of its chunks it takes the rows one at a time, a
        // sweep over the row in shared memory for its amax (shuffles), its
        // scale, then a second sweep that writes its codes with the rowwise
        // quantiser's arithmetic; after the chunk it counts the rows as done
        // for their 128-row blocks (release) and hands the buffer back. No
        // warp waits for another warp's rows and nothing here waits on another
        // CTA; a chunk is only ever claimed by a running CTA, so every counted
        // row block completes, and the GEMM below waits only for those counts.
        if (warp == 0 && lane == 0) {
            const int R = args.qg_rows;
            // Chunks are claimed kQgClaim at a time; the next batch is claimed
            // halfway through staging the current one, so the atomic's round
            // trip overlaps the copies.
            int cur = (int)atomicAdd(args.qg_ctr, (uint32_t)kQgClaim);
            int nxt = 0;
            int k = 0;      // chunks of the current batch staged so far
            int stop = 0;   // buffers that have been given the end mark
            for (int it = 0; stop < kQgBufs; ++it) {
                const int b = it % kQgBufs;
                if (!mbar_wait_bounded(&qempty[b], (uint32_t)((it / kQgBufs) & 1) ^ 1u, abort_flag, args.err)) {
                    // Give up: mark every buffer, waiting for none of them.
                    for (int q = 0; q < kQgBufs; ++q) qchunk[q] = -1;
                    for (int q = 0; q < kQgBufs; ++q) mbar_arrive(&qfull[q]);
                    break;
                }
                const int c = cur + k;
                if (c >= args.qg_chunks) {
                    qchunk[b] = -1;  // no rows left: warp b stops at this buffer
                    mbar_arrive(&qfull[b]);
                    ++stop;
                    continue;
                }
                const int r0 = c * R;
                const int rows = args.M - r0 < R ? args.M - r0 : R;
                const uint32_t bytes = (uint32_t)rows * (uint32_t)args.K * 2u;
                qchunk[b] = c;
                mbar_arrive_expect_tx(&qfull[b], bytes);
                bulk_load_g2s(smem + (size_t)b * kQgBufBytes, args.qg_a + (size_t)r0 * args.K, bytes, &qfull[b]);
                if (++k == kQgClaim / 2) nxt = (int)atomicAdd(args.qg_ctr, (uint32_t)kQgClaim);
                if (k == kQgClaim) {
                    cur = nxt;
                    k = 0;
                }
            }
        } else if (warp >= 2) {
            const int w = warp - 2;  // owns staging buffer w
            const int R = args.qg_rows;
            const int K = args.K;
            const int nvec = K >> 3;
            for (int j = 0;; ++j) {
                const bool ok = mbar_wait_bounded(&qfull[w], (uint32_t)(j & 1), abort_flag, args.err);
                const int c = ok ? qchunk[w] : -1;
                if (!__all_sync(0xffffffffu, c >= 0)) break;  // no more rows (or an expired wait)
                const int r0 = c * R;
                const int rows = args.M - r0 < R ? args.M - r0 : R;
                for (int lr = 0; lr < rows; ++lr) {
                    const int64_t row = (int64_t)r0 + lr;
                    const uint4* src =
                        reinterpret_cast<const uint4*>(smem + (size_t)w * kQgBufBytes + (size_t)lr * K * 2);
                    uint32_t packed = 0;
#pragma unroll 4
                    for (int vi = lane; vi < nvec; vi += 32) packed = absmax8(src[vi], packed);
                    uint32_t m = fold_halves(packed);
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
                    const ScaleCtx sc = scale_ctx<FP8DIT_E4M3FN>(bf16_bits_to_float(m));
                    const Quot2 q2 = quot2_of(sc);
                    uint2* dst = reinterpret_cast<uint2*>(args.qg_q + row * K);
                    if (sc.fast) {
#pragma unroll 4
                        for (int vi = lane; vi < nvec; vi += 32) dst[vi] = quant8<FP8DIT_E4M3FN, true>(src[vi], q2);
                    } else {
                        for (int vi = lane; vi < nvec; vi += 32) dst[vi] = quant8<FP8DIT_E4M3FN, false>(src[vi], q2);
                    }
                    if (lane == 0) args.qg_s[row] = sc.s;
                }
                // The chunk's codes and scales, then its counts; the staged rows
                // have been read (generic proxy) before the copy engine (async
                // proxy) refills the buffer.
                __threadfence();
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    for (int r = r0; r < r0 + rows;) {
                        const int blk = r >> 7;
                        const int e = (blk + 1) * 128 < r0 + rows ? (blk + 1) * 128 : r0 + rows;
                        red_add_release_gpu_u32(args.qg_ctr + 2 + blk, (uint32_t)(e - r));
                        r = e;
                    }
                    mbar_arrive(&qempty[w]);
                }
            }
        }
        // The operand ring is the GEMM's from here on.
        __syncthreads();
    }

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            int64_t armed = 0;
            SegSched ss = seg_begin(args, unit, units, C::SPLIT_OK);
            Segment sg;
            while (!aborted && seg_next(ss, sg)) {
                const TileCoord tc = tile_coord(args, sg.t);
                const int a_row = tc.tm * C::BM + (int)rank * C::ROWS;
                const int b_row = tc.tn * BN + (int)rank * C::B_ROWS;
                if constexpr (C::QG) {
                    // This CTA's 128 rows of A must be quantised (phase Q of
                    // some running CTA) before their codes are loaded.
                    const int need = args.M - a_row < C::ROWS ? args.M - a_row : C::ROWS;
                    if (need > 0 && !wait_count_bounded(args.qg_ctr + 2 + (a_row >> 7), (uint32_t)need, abort_flag,
                                                        args.err)) {
                        aborted = true;
                        abort_peer();
                        break;
                    }
                    fence_proxy_async_global();  // the acquired codes, before the copies read them
                }
                for (int kb = sg.k0; kb < sg.k1; ++kb) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, args.err)) {
                        aborted = true;
                        abort_peer();
                        break;
                    }
                    if (CONV) {
                        // Each CTA tracks its own A and W loads; its converter
                        // warps wait on them. W8: the codes go to the upper half
                        // of the B buffer (decoded in place).
                        mbar_arrive_expect_tx(&full[stage], C::TX_BYTES);
                        tma_load_2d(sA + stage * C::A_STAGE, &args.tmA, &full[stage], kb * C::KE, a_row);
                        tma_load_2d(sB + stage * C::B_BYTES + (W8 ? C::RAW_BYTES : 0), &args.tmB[tc.g], &full[stage],
                                    kb * C::KE, b_row);
                    } else if (CG == 2) {
                        const uint32_t bar = mapa_shared(smem_u32(&full[stage]), 0);
                        if (leader) mbar_arrive_expect_tx(&full[stage], CG * C::TX_BYTES);
                        tma_load_2d_pair(sA + stage * C::A_STAGE, &args.tmA, bar, kb * C::KE, a_row);
                        tma_load_2d_pair(sB + stage * C::B_BYTES, &args.tmB[tc.g], bar, kb * C::KE, b_row);
                    } else {
                        // Single CTA: A brings args.a_box_rows rows (M < 128) or 128.
                        mbar_arrive_expect_tx(&full[stage], args.a_box_rows * C::ROW_BYTES + C::B_BYTES);
                        tma_load_2d(sA + stage * C::A_STAGE, &args.tmA, &full[stage], kb * C::KE, a_row);
                        tma_load_2d(sB + stage * C::B_BYTES, &args.tmB[tc.g], &full[stage], kb * C::KE, b_row);
                    }
                    ++armed;
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (aborted && (leader || CONV)) {
                // Let every copy signalled on this CTA's barriers land before exit.
                for (int s = 0; s < C::STAGES; ++s) {
                    if (armed <= s) break;
                    const int64_t last = s + (int64_t)C::STAGES * ((armed - 1 - s) / C::STAGES);
                    mbar_wait_bounded(&full[s], (uint32_t)((last / C::STAGES) & 1), nullptr, args.err);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (pair leader)
        if (lane == 0 && leader) {
            constexpr uint32_t idesc = W8 ? umma_idesc_bf16_f32(C::BM, BN) : umma_idesc_e4m3_f32(C::BM, BN);
            uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
            SegSched ss = seg_begin(args, unit, units, C::SPLIT_OK);
            Segment sg;
            while (!aborted && seg_next(ss, sg)) {
                if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag, args.err)) {
                    aborted = true;
                    abort_peer();
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * BN;
                for (int kb = sg.k0; kb < sg.k1; ++kb) {
                    // W8: both CTAs' converted operands (and, through the
                    // converters' waits, both CTAs' loads) are ready. FP8: both
                    // CTAs' TMA loads landed.
                    if (!mbar_wait_bounded(CONV ? &conv[stage] : &full[stage], phase, abort_flag, args.err)) {
                        aborted = true;
                        abort_peer();
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sA + stage * C::A_STAGE);
                    const uint32_t b0 = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
                    for (int j = 0; j < C::ROW_BYTES / 32; ++j) {  // 32 bytes of K per MMA
                        const uint64_t ad = umma_desc_kmajor_sw128(a0 + 32 * j);
                        const uint64_t bd = umma_desc_kmajor_sw128(b0 + 32 * j);
                        const uint32_t accum = (kb > sg.k0 || j > 0) ? 1u : 0u;  // a segment starts a new sum
                        if (W8) {
                            if (CG == 2) mma_bf16_pair(d_tmem, ad, bd, idesc, accum);
                            else mma_bf16(d_tmem, ad, bd, idesc, accum);
                        } else {
                            if (CG == 2) mma_f8f6f4_pair(d_tmem, ad, bd, idesc, accum);
                            else mma_f8f6f4(d_tmem, ad, bd, idesc, accum);
                        }
                    }
                    // The ring slot is free (in both CTAs) once these MMAs have read it.
                    if (CG == 2) mma_commit_pair_multicast(&empty[stage], 0x3);
                    else mma_commit(&empty[stage]);
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (aborted) break;
                if (CG == 2) mma_commit_pair_multicast(&tfull[acc], 0x3);
                else mma_commit(&tfull[acc]);
                if (++acc == C::ACC) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            // Every MMA this thread issued has completed once `drain` fires.
            if (CG == 2) mma_commit_pair(drain);
            else mma_commit(drain);
            mbar_wait_bounded(drain, 0, nullptr, args.err);
        }
        __syncwarp();
    } else if (warp < 2 + C::EPI_WARPS) {
        // ------------------------------------------------ epilogue warps
        const int q = warp & 3;          // TMEM lane quarter this warp may access
        const int ew = warp - 2;         // 0..7
        const int col0 = (ew >> 2) * C::EPI_COLS;  // this warp's half of the tile's columns
        uint8_t* stg = staging + ew * C::STG_BYTES;
        float* sw_s = swb + ew * C::SWB_FLOATS;
        float* b_s = sw_s + C::EPI_COLS;
        constexpr int SW_V4 = (C::EPI_COLS / 4 + 31) / 32;  // float4 of sw per lane
        constexpr int B_V8 = (C::EPI_COLS / 8 + 31) / 32;   // 8-wide bf16 bias vectors per lane

        // Per-tile epilogue operands, fetched one tile ahead: the scales and
        // bias of this warp's columns, and sa of this lane's row. All loads of
        // a tile are independent, so one memory round trip covers them, and
        // it overlaps the previous tile's processing.
        struct Pre {
            float4 sw[SW_V4];
            uint4 b[B_V8];
            float sa;
        };
        auto fetch = [&](int t, Pre& p) {
            const TileCoord tc = tile_coord(args, t);
            const GemmProblem& P = args.prob[tc.g];
#pragma unroll
            for (int i = 0; i < SW_V4; ++i) {
                const int v = i * 32 + lane;
                const int n = tc.tn * BN + col0 + v * 4;
                p.sw[i] = (v < C::EPI_COLS / 4 && n < P.N) ? __ldg(reinterpret_cast<const float4*>(P.sw + n))
                                                            : make_float4(0, 0, 0, 0);
            }
#pragma unroll
            for (int i = 0; i < B_V8; ++i) {
                const int v = i * 32 + lane;
                const int n = tc.tn * BN + col0 + v * 8;
                p.b[i] = (v < C::EPI_COLS / 8 && n < P.N && P.bias != nullptr)
                             ? __ldg(reinterpret_cast<const uint4*>(P.bias + n))
                             : make_uint4(0, 0, 0, 0);
            }
            const int row = tc.tm * C::BM + (int)rank * C::ROWS + q * 32 + lane;
            // Fused linear: the launch itself writes sa, so it is read after
            // the tile's accumulator is ready (below), not ahead.
            p.sa = (row < args.M && !C::QG) ? (args.sa != nullptr ? __ldg(args.sa + row) : 1.0f) : 0.0f;
        };
        auto publish = [&](const Pre& p) {  // this warp's smem copy of sw / bias (fp32)
#pragma unroll
            for (int i = 0; i < SW_V4; ++i) {
                if (i * 32 + lane >= C::EPI_COLS / 4) break;
                *reinterpret_cast<float4*>(sw_s + (i * 32 + lane) * 4) = p.sw[i];
            }
#pragma unroll
            for (int i = 0; i < B_V8; ++i) {
                if (i * 32 + lane >= C::EPI_COLS / 8) break;
                const uint32_t w[4] = {p.b[i].x, p.b[i].y, p.b[i].z, p.b[i].w};
                float* dst = b_s + (i * 32 + lane) * 8;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    dst[2 * k] = __uint_as_float(w[k] << 16);
                    dst[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
                }
            }
        };

        // Split-K: the CTA whose arrival completes tile t's count adds, for
        // every valid row of the tile, the S partials in piece order (the same
        // order whichever piece arrives last, so results are deterministic),
        // applies the epilogue and stores bf16 to y. The tile goes one 32-row
        // quarter at a time: one thread bulk-copies that quarter of every
        // piece's partial block ([quarter][column part][float4][row lane],
        // 16 KB contiguous per piece) into the operand ring, which is idle by
        // now (one segment per CTA), so the copy engine keeps the whole
        // quarter in flight; then each thread sums float4 i of the S copies.
        auto split_reduce = [&](int t) {
            const TileCoord tc = tile_coord(args, t);
            const GemmProblem& P = args.prob[tc.g];
            const int r0 = tc.tm * C::BM;
            const int rows = args.M - r0 < C::BM ? args.M - r0 : C::BM;
            const int c0 = tc.tn * BN;
            const int S = args.split_k;
            constexpr uint32_t QBYTES = 32 * BN * 4;              // one quarter of one piece
            constexpr int QF4 = (int)(QBYTES / 16);
            constexpr size_t PIECE4 = (size_t)C::ROWS * BN / 4;   // float4 per piece
            const float4* src = reinterpret_cast<const float4*>(args.sk_partial) + (size_t)t * S * PIECE4;
            const float4* buf = reinterpret_cast<const float4*>(smem);
            const int nq = (rows + 31) >> 5;
            for (int qq = 0; qq < nq; ++qq) {
                if (ew == 0 && lane == 0) {
                    bool ok = *abort_flag == 0;
                    if (ok) {
                        if (qq == 0) fence_proxy_async_global();  // the acquired partials, before the copies
                        mbar_arrive_expect_tx(redbar, (uint32_t)S * QBYTES);
                        for (int p = 0; p < S; ++p)
                            bulk_load_g2s(smem + (size_t)p * QBYTES, src + (size_t)p * PIECE4 + (size_t)qq * QF4,
                                          QBYTES, redbar);
                        ok = mbar_wait_bounded(redbar, (uint32_t)(qq & 1), abort_flag, args.err);
                    }
                    *split_ok = ok ? 1u : 0u;
                }
                named_barrier_sync(1, 32 * C::EPI_WARPS);
                if (*split_ok != 1u) break;  // uniform: every epilogue thread reads the same word
                for (int i = ew * 32 + lane; i < QF4; i += 32 * C::EPI_WARPS) {
                    const int r = qq * 32 + (i & 31);
                    const int f = i >> 5;  // float4 column of the tile
                    const int n = c0 + 4 * f;
                    if (r >= rows || n >= P.N) continue;
                    float4 v = buf[i];
#pragma unroll
                    for (int p = 1; p < kSplitMaxPieces; ++p) {
                        if (p < S) {
                            const float4 x = buf[p * QF4 + i];
                            v.x += x.x;
                            v.y += x.y;
                            v.z += x.z;
                            v.w += x.w;
                        }
                    }
                    const float sa = args.sa != nullptr ? __ldg(args.sa + r0 + r) : 1.0f;
                    const float4 w4 = __ldg(reinterpret_cast<const float4*>(P.sw + n));
                    uint2 b2 = make_uint2(0u, 0u);
                    if (P.bias != nullptr) b2 = __ldg(reinterpret_cast<const uint2*>(P.bias + n));
                    const float o0 = fmaf(v.x * sa, w4.x, __uint_as_float(b2.x << 16));
                    const float o1 = fmaf(v.y * sa, w4.y, __uint_as_float(b2.x & 0xffff0000u));
                    const float o2 = fmaf(v.z * sa, w4.z, __uint_as_float(b2.y << 16));
                    const float o3 = fmaf(v.w * sa, w4.w, __uint_as_float(b2.y & 0xffff0000u));
                    *reinterpret_cast<uint2*>(P.y + (size_t)(r0 + r) * P.N + n) =
                        make_uint2(pack_bf16x2(o0, o1), pack_bf16x2(o2, o3));
                }
                named_barrier_sync(1, 32 * C::EPI_WARPS);  // every thread is done with the staged quarter
            }
        };

        uint32_t acc = 0, acc_phase = 0;
        uint32_t stores = 0;
        const bool split = C::SPLIT_OK && args.split_k > 1;
        Pre pre;
        SegSched ss = seg_begin(args, unit, units, C::SPLIT_OK);
        SegSched look = ss;  // one segment ahead, for the operand prefetch
        Segment sg, nx;
        bool has_next = seg_next(look, nx);
        if (has_next) fetch(nx.t, pre);
        while (seg_next(ss, sg)) {
            has_next = seg_next(look, nx);
            const TileCoord tc = tile_coord(args, sg.t);
            __syncwarp();  // every lane is done reading the previous tile's copy
            publish(pre);
            float sa = pre.sa;
            __syncwarp();
            if (has_next) fetch(nx.t, pre);
            const int row0 = tc.tm * C::BM + (int)rank * C::ROWS + q * 32;  // first row of this warp's box
            // Stream-K roles of this segment: a tail stores its fp32 partial for
            // the unit that finishes the tile; a head adds that partial. A warp's
            // partial (32 rows x EPI_COLS fp32) is stored lane-fastest: float4 v
            // of row `lane` in column chunk c sits at [(c * 8 + v) * 32 + lane],
            // so every warp access moves 512 contiguous bytes.
            const bool tail = !split && sg.k0 > 0;
            const bool head = !split && sg.k0 == 0 && sg.k1 < args.num_kb;
            // Stream-K: a tile split between units u (head: the tile's start, u's
            // last segment) and u + 1 (tail: the tile's end, u + 1's first
            // segment) is finished by whichever of the two warps arrives
            // second, so neither ever waits for the other. Per epilogue warp
            // one flag word F: 0 = nothing stored, 1 = the tail's partial is
            // stored, 2 = the head's partial is stored. The tail stores its
            // partial and swaps in 1; the head, if F already reads 1, finishes
            // at once, else stores its own partial and swaps in 2. A swap that
            // returns the other side's mark makes this warp the finisher: it
            // adds the other partial to its own accumulator (fp32 addition
            // commutes, so the result does not depend on which side finishes),
            // applies the epilogue, stores y and clears F for the next launch.
            const size_t part_elems = 32 * C::EPI_COLS;
            uint32_t* sk_f = nullptr;
            const float4* tail_part = nullptr;  // partials of the split tile this warp shares
            const float4* head_part = nullptr;
            if (tail || head) {
                const int slot = tail ? unit : unit + 1;  // indexed by the tail's unit
                const size_t idx = ((size_t)slot * 2 + rank) * C::EPI_WARPS + ew;
                tail_part = reinterpret_cast<const float4*>(args.sk_partial + idx * part_elems) + lane;
                head_part = reinterpret_cast<const float4*>(args.sk_partial_head + idx * part_elems) + lane;
                sk_f = args.sk_flag + idx;
            }
            // Mode of the next pass over the accumulator: store it raw to
            // `mine`, or add `theirs` (prefetched chunk by chunk into pp) and
            // run the epilogue, or (neither) just the epilogue.
            float4* mine = tail ? const_cast<float4*>(tail_part) : nullptr;
            const float4* theirs = nullptr;
            float4 pp[8];  // the other side's partial for the next column chunk
            if (head) {
                uint32_t f = 0;
                if (lane == 0) f = ld_acquire_gpu_u32(sk_f);
                f = __shfl_sync(0xffffffffu, f, 0);
                __syncwarp();  // lane 0's acquire orders every lane's partial loads
                if (f == 1u) {
                    theirs = tail_part;  // the tail's partial is there: finish now
#pragma unroll
                    for (int v = 0; v < 8; ++v) pp[v] = __ldcg(theirs + v * 32);
                } else {
                    mine = const_cast<float4*>(head_part);  // store ours; the tail may finish
                }
            }

            // Every lane waits; the warp then agrees (and reconverges) before
            // the warp-collective TMEM loads.
            const bool ready = mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, args.err);
            bool failed = false;
            if (!__all_sync(0xffffffffu, ready)) {
                if (lane == 0) abort_peer();
                if (!split) break;
                failed = true;  // split-K: still meet the CTA's epilogue barriers below
            }
            if constexpr (C::QG) {
                // This lane's row was counted as quantised before the producer
                // loaded its codes; acquire that count here too, then read sa.
                const int row = row0 + lane;
                if (row < args.M) {
                    (void)ld_acquire_gpu_u32(args.qg_ctr + 2 + (row >> 7));
                    sa = __ldcg(args.sa + row);
                }
            }
            tc_fence_after();
            const int n_tile = args.prob[tc.g].N;
            const uint32_t t_addr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN + col0;
            // One 16-column half of 32-column chunk c, its accumulator in r:
            // split-K pieces and stream-K partials store it raw; otherwise (a
            // stream-K finisher first adds the other side's partial) scale,
            // bias, bf16 and half of row `lane` of the chunk's 32 x 32 staging
            // box (64-byte rows, 64-byte swizzle).
            auto half = [&](int c, int hh, uint32_t(&r)[16]) {
                if (split) {
                    // This piece's raw fp32 partial, [q][column part][float4][lane]:
                    // every warp store moves 512 contiguous bytes. Warps whose
                    // rows all lie past M store nothing (nothing reads them).
                    if (row0 < args.M) {
                        float4* dst = reinterpret_cast<float4*>(args.sk_partial) +
                                      (size_t)((int64_t)sg.t * args.split_k + sg.piece) * (C::ROWS * BN / 4) +
                                      ((((size_t)q * C::HALVES + (ew >> 2)) * (C::EPI_COLS / 4) + c * 8 + hh * 4) << 5) +
                                      lane;
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            __stcg(dst + v * 32,
                                   make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                               __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3])));
                    }
                    return;
                }
                if (mine != nullptr) {
                    // Raw fp32 accumulator: row `lane`, columns c*32 + hh*16 ..+15,
                    // lane-fastest (every warp store moves 512 contiguous bytes).
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        __stcg(mine + (c * 8 + hh * 4 + v) * 32,
                               make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                           __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3])));
                    return;
                }
                if (theirs != nullptr) {
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        r[4 * v] = __float_as_uint(__uint_as_float(r[4 * v]) + pp[hh * 4 + v].x);
                        r[4 * v + 1] = __float_as_uint(__uint_as_float(r[4 * v + 1]) + pp[hh * 4 + v].y);
                        r[4 * v + 2] = __float_as_uint(__uint_as_float(r[4 * v + 2]) + pp[hh * 4 + v].z);
                        r[4 * v + 3] = __float_as_uint(__uint_as_float(r[4 * v + 3]) + pp[hh * 4 + v].w);
                    }
                }
                uint32_t packed[8];
#pragma unroll
                for (int j = 0; j < 16; j += 4) {
                    const float4 w4 = *reinterpret_cast<const float4*>(sw_s + c * 32 + hh * 16 + j);
                    const float4 b4 = *reinterpret_cast<const float4*>(b_s + c * 32 + hh * 16 + j);
                    const float o0 = fmaf(__uint_as_float(r[j + 0]) * sa, w4.x, b4.x);
                    const float o1 = fmaf(__uint_as_float(r[j + 1]) * sa, w4.y, b4.y);
                    const float o2 = fmaf(__uint_as_float(r[j + 2]) * sa, w4.z, b4.z);
                    const float o3 = fmaf(__uint_as_float(r[j + 3]) * sa, w4.w, b4.w);
                    packed[j / 2] = pack_bf16x2(o0, o1);
                    packed[j / 2 + 1] = pack_bf16x2(o2, o3);
                }
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const int phys = (hh * 2 + k) ^ ((lane >> 1) & 3);
                    *reinterpret_cast<uint4*>(stg + lane * 64 + phys * 16) =
                        make_uint4(packed[4 * k], packed[4 * k + 1], packed[4 * k + 2], packed[4 * k + 3]);
                }
            };
            // Chunks this warp holds (warp-uniform; fewer where the tile passes N).
            const int base_n = tc.tn * BN + col0;
            int nch = failed ? 0 : (n_tile - base_n + 31) / 32;
            if (nch > C::EPI_COLS / 32) nch = C::EPI_COLS / 32;
            if (nch < 0) nch = 0;
            // Two 16-register buffers: the TMEM load of the next half is in
            // flight while the current half is processed.
            // Pass 0 over the accumulator; a stream-K warp that learns after
            // publishing its partial that it finishes the tile makes pass 1.
            bool finish = false;
#pragma unroll 1
            for (int pass = 0; pass < 2; ++pass) {
                uint32_t ra[16], rb[16];
                if (nch > 0) tmem_ld_32x32b_x16(t_addr, ra);
#pragma unroll 1
                for (int c = 0; c < nch; ++c) {
                    const int n0 = base_n + c * 32;
                    tmem_wait_ld16(ra);
                    tmem_ld_32x32b_x16(t_addr + c * 32 + 16, rb);
                    const bool store = !split && mine == nullptr;
                    // The single staging buffer is free once the previous store has read it.
                    if (store && stores >= 1) {
                        if (lane == 0) bulk_wait_group_read<0>();
                        __syncwarp();
                    }
                    half(c, 0, ra);
                    tmem_wait_ld16(rb);
                    if (c + 1 < nch) tmem_ld_32x32b_x16(t_addr + (c + 1) * 32, ra);
                    half(c, 1, rb);
                    if (theirs != nullptr && c + 1 < C::EPI_COLS / 32) {
                        // Next chunk's partial, in flight while this chunk is stored.
#pragma unroll
                        for (int v = 0; v < 8; ++v) pp[v] = __ldcg(theirs + ((c + 1) * 8 + v) * 32);
                    }
                    if (!store) continue;
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0 && row0 < args.M) {
                        tma_store_2d(&args.tmY[tc.g], stg, n0, row0);
                        bulk_commit_group();
                    }
                    ++stores;
                }
                if (pass == 1 || !(tail || head) || failed) break;
                finish = theirs != nullptr;  // a head that found the tail's partial
                if (mine == nullptr) break;
                // Publish the partial (every lane's stores, then the mark) and
                // learn whether the other side has already been here.
                __threadfence();
                __syncwarp();
                uint32_t old = 0;
                if (lane == 0) old = atom_exch_acq_rel_gpu_u32(sk_f, tail ? 1u : 2u);
                old = __shfl_sync(0xffffffffu, old, 0);
                __syncwarp();  // lane 0's acquire orders every lane's partial loads
                finish = old == (tail ? 2u : 1u);
                if (!finish) break;
                mine = nullptr;  // pass 1: add the other side's partial, epilogue, y
                theirs = tail ? head_part : tail_part;
#pragma unroll
                for (int v = 0; v < 8; ++v) pp[v] = __ldcg(theirs + v * 32);
            }
            if (finish) {
                // This warp finished the split tile: clear the mark, so the
                // workspace is ready for the next launch without a host reset
                // (stream-ordered launches and graph replays included).
                __syncwarp();
                if (lane == 0) *sk_f = 0u;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (CG == 2) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
                else mbar_arrive(&tempty[acc]);
            }
            if (++acc == C::ACC) {
                acc = 0;
                acc_phase ^= 1u;
            }
            if (split) {
                // Every thread fences its partial stores; after the barrier
                // thread 0 arrives on the tile's counter (acquire-release).
                // The arrival that completes the count sees every piece's
                // partial, resets the counter for the next launch and reduces
                // the whole tile; every other piece is done. No piece ever
                // waits for another, so nothing depends on the pieces being
                // resident at the same time (other kernels may hold SMs). A
                // piece whose accumulator wait expired does not arrive: its
                // tile stays unreduced and the device error word reports it.
                uint32_t* arrive = args.split_arrive + sg.t;
                if (failed && lane == 0) *split_fail = 1u;
                __threadfence();
                named_barrier_sync(1, 32 * C::EPI_WARPS);
                if (ew == 0 && lane == 0) {
                    uint32_t last = 0u;
                    if (*split_fail == 0u && atom_acq_rel_gpu_add_u32(arrive, 1u) == (uint32_t)args.split_k - 1u) {
                        *arrive = 0u;
                        last = 1u;
                    }
                    *split_ticket = last;
                }
                named_barrier_sync(1, 32 * C::EPI_WARPS);
                if (*split_ticket == 1u) {
                    if constexpr (C::SPLIT_OK) split_reduce(sg.t);
                }
            }
        }
        if (lane == 0) bulk_wait_group<0>();  // all output stores complete
        __syncwarp();
    } else {
        // ------------------------------------------------ FP8 -> bf16 weight decoders (W8)
        // Decoder warp s owns ring stage s, so it waits on that stage's
        // barrier phase after phase, and STAGES stages are decoded, fenced and
        // released concurrently. The stage's B buffer (B_ROWS rows of 128
        // bytes) holds, in its upper half, the FP8 codes as loaded (B_ROWS
        // rows of 64 bytes). They are decoded in place into B_ROWS rows x 64
        // bf16 with the 128-byte swizzle (16-byte chunk c of row r at chunk
        // c ^ (r & 7)), the K-major layout the MMA descriptors describe; E4M3
        // values are exact in bf16. Rows go in batches of kRowsPerBatch, each
        // read whole before any of it is written: writing decoded rows
        // [r0, r1) covers code rows below 2 * r1 - B_ROWS <= r1, all read
        // already, so no code is overwritten before it is decoded.
        if constexpr (W8) {
            constexpr int kIters = 4;                      // 16-byte code chunks per lane per batch
            constexpr int kRowsPerBatch = kIters * 32 / 4;  // 4 chunks per 64-byte code row
            const int own = warp - (2 + C::EPI_WARPS);     // the stage this warp decodes
            uint32_t stage = 0, phase = 0;
            bool stop = false;
            SegSched ss = seg_begin(args, unit, units, C::SPLIT_OK);
            Segment sg;
            while (!stop && seg_next(ss, sg)) {
                for (int kb = sg.k0; kb < sg.k1; ++kb) {
                    if ((int)stage == own) {
                        const bool ok = mbar_wait_bounded(&full[stage], phase, abort_flag, args.err);
                        if (!__all_sync(0xffffffffu, ok)) {
                            if (lane == 0) abort_peer();
                            stop = true;
                            break;
                        }
                        uint8_t* dst = sB + stage * C::B_BYTES;
                        const uint8_t* raw = dst + C::RAW_BYTES;
#pragma unroll 1
                        for (int r0 = 0; r0 < C::B_ROWS; r0 += kRowsPerBatch) {
                            uint4 v[kIters];
#pragma unroll
                            for (int i = 0; i < kIters; ++i)
                                v[i] = *reinterpret_cast<const uint4*>(raw + r0 * 64 + (i * 32 + lane) * 16);
                            __syncwarp();  // the whole batch is read before any lane writes
#pragma unroll
                            for (int i = 0; i < kIters; ++i) {
                                const int r = r0 + ((i * 32 + lane) >> 2), c = lane & 3;
                                const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
                                uint32_t o[8];
#pragma unroll
                                for (int k = 0; k < 4; ++k) {
                                    const __half2_raw lo =
                                        __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[k] & 0xffffu), __NV_E4M3);
                                    const __half2_raw hi =
                                        __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[k] >> 16), __NV_E4M3);
                                    o[2 * k] = pack_bf16x2(__half2float(__ushort_as_half(lo.x)),
                                                           __half2float(__ushort_as_half(lo.y)));
                                    o[2 * k + 1] = pack_bf16x2(__half2float(__ushort_as_half(hi.x)),
                                                               __half2float(__ushort_as_half(hi.y)));
                                }
                                *reinterpret_cast<uint4*>(dst + r * 128 + (((2 * c) ^ (r & 7)) << 4)) =
                                    make_uint4(o[0], o[1], o[2], o[3]);
                                *reinterpret_cast<uint4*>(dst + r * 128 + (((2 * c + 1) ^ (r & 7)) << 4)) =
                                    make_uint4(o[4], o[5], o[6], o[7]);
                            }
                        }
                        fence_proxy_async_smem();  // the tensor core reads these bytes through the async proxy
                        __syncwarp();
                        if (lane == 0) {
                            if (CG == 2) mbar_arrive_cluster(mapa_shared(smem_u32(&conv[stage]), 0));
                            else mbar_arrive(&conv[stage]);
                        }
                    }
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
        __syncwarp();
    }

    if (*abort_flag) {
        // Give copies that this CTA cannot wait for (a pair's follower signals
        // the leader's barriers) time to land before shared memory is released.
        const unsigned long long t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 50000ull) {
        }
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (C::QG) {
        // The CTA that finishes last returns the fused linear's counters to
        // zero for the next launch (no other CTA reads them any more).
        if (threadIdx.x == 0) {
            __threadfence();
            *qlast = atomicAdd(args.qg_ctr + 1, 1u) == gridDim.x - 1 ? 1u : 0u;
        }
        __syncthreads();
        if (*qlast) {
            const int nrb = (args.M + 127) >> 7;
            for (int i = threadIdx.x; i < 2 + nrb; i += blockDim.x) args.qg_ctr[i] = 0u;
        }
    }
    if (CG == 2) cluster_sync_all();  // both CTAs done with TMEM and each other's barriers
    if (warp == 1) {
        tc_fence_after();
        if (CG == 2) tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
        else tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

template <int CG, int BN, int OPS>
cudaError_t launch_cfg(const GemmArgs& args, int units, cudaStream_t stream) {
    using C = Cfg<CG, BN, OPS>;
    static bool attr_done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 64 && !attr_done[dev]) {
        e = cudaFuncSetAttribute(gemm_e4m3_kernel<CG, BN, OPS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_done[dev] = true;
    }
    return launch_pdl(gemm_e4m3_kernel<CG, BN, OPS>, dim3((unsigned)(units * CG)), dim3(C::THREADS), C::SMEM_BYTES,
                      stream, CG, args);
}

}  // namespace

int gemm_cta_group(int cfg) {
    return (cfg == kCfgPair256 || cfg == kCfgW8Pair256 || cfg == kCfgQGPair256) ? 2 : 1;
}
int gemm_block_m(int cfg) { return 128 * gemm_cta_group(cfg); }
int gemm_block_n(int cfg) {
    return cfg == kCfg128x64 ? 64 : (cfg == kCfg128x128 || cfg == kCfgW8128x128 || cfg == kCfgQG128x128) ? 128 : 256;
}
int gemm_b_box_rows(int cfg) { return cfg == kCfg128x256 ? 256 : cfg == kCfg128x64 ? 64 : 128; }
bool gemm_weight_only(int cfg) { return cfg == kCfgW8Pair256 || cfg == kCfgW8128x128; }
bool gemm_quantizes_a(int cfg) { return cfg == kCfgQGPair256 || cfg == kCfgQG128x128; }
int gemm_k_elems(int cfg) { return gemm_weight_only(cfg) ? 64 : 128; }

// MMA units (CTA pairs or CTAs) to launch: one per tile, at most one per SM (pair).
int gemm_units_for(int cfg, int num_tiles, const DeviceInfo* dev) {
    const int max_units = dev->num_sms / gemm_cta_group(cfg);
    return num_tiles < max_units ? num_tiles : max_units;
}

cudaError_t launch_gemm(int cfg, const GemmArgs& args, int units, cudaStream_t stream) {
    switch (cfg) {
        case kCfgPair256:
            return launch_cfg<2, 256, kOpsFp8>(args, units, stream);
        case kCfg128x256:
            return launch_cfg<1, 256, kOpsFp8>(args, units, stream);
        case kCfg128x128:
            return launch_cfg<1, 128, kOpsFp8>(args, units, stream);
        case kCfgW8Pair256:
            return launch_cfg<2, 256, kOpsW8>(args, units, stream);
        case kCfgW8128x128:
            return launch_cfg<1, 128, kOpsW8>(args, units, stream);
        case kCfgQGPair256:
            return launch_cfg<2, 256, kOpsQG>(args, units, stream);
        case kCfgQG128x128:
            return launch_cfg<1, 128, kOpsQG>(args, units, stream);
        case kCfg128x64:
            return launch_cfg<1, 64, kOpsFp8>(args, units, stream);
        default:
            return cudaErrorInvalidValue;
    }
}

}  // namespace fp8dit
