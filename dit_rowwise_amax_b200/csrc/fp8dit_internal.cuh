// Internal declarations and sm_100a device helpers shared by the fp8dit
// kernels: mbarriers, TMA (no multicast anywhere), tcgen05 / TMEM, and the
// bounded wait every spin in the library goes through.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "../../include/fp8dit.h"

namespace fp8dit {

// ------------------------------------------------------------------ errors
// Bits of the per-device error word.
enum : uint32_t {
    kDevErrTimeout = 1u,
};

// Where a kernel reports an expired wait, and how long a wait may last.
struct DevErr {
    uint32_t* word;
    unsigned long long limit_ns;
};

constexpr unsigned long long kDefaultWaitLimitNs = 2000000000ull;  // 2 s

// ------------------------------------------------------------- host side
// Per-device facts, fetched once per device.
struct DeviceInfo {
    int num_sms;
    int max_smem_optin;
    uint32_t* err_word;  // device address of the library's error word
};

// Returns nullptr (and sets the last error) on failure. Uses the current device.
const DeviceInfo* device_info();
void set_error(const char* fmt, ...);
fp8dit_status cuda_fail(cudaError_t e, const char* what);

// Reduction length K and CUDA device of a linear layer handle.
int64_t linear_k(const fp8dit_linear_s* h);
int linear_device(const fp8dit_linear_s* h);

// cuTensorMapEncodeTiled through the runtime's driver entry point: a 2-D
// row-major tensor of 1- or 2-byte elements (inner = contiguous extent).
fp8dit_status encode_tma_2d(CUtensorMap* map, int elem_bytes, const void* base, uint64_t inner, uint64_t outer,
                            uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                            CUtensorMapSwizzle swizzle);

// Launchers (each validates nothing; the API layer has done it).
cudaError_t launch_quantize_rows(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int fmt,
                                 uint8_t* q, int64_t ldq, float* scale, cudaStream_t stream,
                                 const DeviceInfo* dev);
cudaError_t launch_act_quantize_rows(const uint16_t* h, int64_t M, int64_t K, int64_t ldh, int act, uint8_t* q,
                                     int64_t ldq, float* scale, uint16_t* g, int64_t ldg, cudaStream_t stream,
                                     const DeviceInfo* dev);

struct PerTensorDevDesc {
    const void* src;
    int64_t numel;
    uint8_t* dst;
    float* scale;
    int32_t src_dtype;  // fp8dit_src_dtype
};
size_t per_tensor_workspace_bytes(int32_t n);
cudaError_t launch_per_tensor(const fp8dit_tensor_desc* host_descs, int32_t n, int fmt, void* ws,
                              cudaStream_t stream, const DeviceInfo* dev, DevErr err);

cudaError_t launch_selftest_wait(cudaStream_t stream, DevErr err);
cudaError_t launch_selftest_quotient(unsigned long long* mismatch, cudaStream_t stream);

// Grouped GEMM: up to kMaxGroups products sharing the quantised A.
constexpr int kMaxGroups = 4;

struct GemmProblem {
    const float* sw;
    const uint16_t* bias;  // may be null
    uint16_t* y;           // bf16 [M, N], row-major (split-K stores it directly)
    int32_t N;
    int32_t tiles_n;
    int32_t tile_start;  // first global tile index of this problem
};

struct alignas(64) GemmArgs {
    CUtensorMap tmA;               // A codes [M, K], box 128 x 128 B, 128-byte swizzle
    CUtensorMap tmB[kMaxGroups];   // W codes [N, K], box rows per configuration
    CUtensorMap tmY[kMaxGroups];   // y bf16 [M, N], box 32 x 32, 64-byte swizzle (TMA store)
    GemmProblem prob[kMaxGroups];
    const float* sa;
    int32_t M, K, G;
    int32_t num_tiles;
    int32_t num_kb;
    DevErr err;
    // Stream-K schedule (pair FP8 configuration only): each MMA unit takes an
    // equal contiguous share of the num_tiles x num_kb k-blocks. A tile split
    // between units u and u+1 is finished by u: u+1 computes its k-block tail
    // first, stores the fp32 partial in sk_partial and sets sk_flag to 1; u
    // waits for 1, adds the partial and clears the flag again.
    int32_t stream_k;
    // Split-K (128 x 128 single-CTA tiles, few tiles): split_k > 1 pieces per
    // tile, CTA u computing piece u % split_k of tile u / split_k over an equal
    // share of the k-blocks. Every piece stores its fp32 partial and arrives on
    // the tile's counter; the arrival that completes the count resets it and
    // its CTA adds the split_k partials in piece order for the whole tile and
    // writes y. No piece waits for another.
    int32_t split_k;
    // Rows of A one TMA load brings per stage in the single-CTA FP8 plans:
    // M rounded up to 8 when M < 128 (one row tile), else 128. The MMA still
    // reads 128 rows; rows past the box hold stale data and only feed
    // accumulator rows past M, which are never stored.
    int32_t a_box_rows;
    uint32_t* split_arrive;  // split-K: arrival counter per tile (zero between launches)
    // Fused linear (quantise, then GEMM, in one launch): bf16 A, written into
    // the FP8 A that tmA describes and the scales sa by the launch itself.
    const uint16_t* qg_a;  // bf16 A [M, K], contiguous
    uint8_t* qg_q;         // its E4M3 codes [M, K] (what tmA describes)
    float* qg_s;           // its per-token scales [M] (== sa)
    uint32_t* qg_ctr;      // [0] chunks claimed, [1] CTAs finished, [2 + b] rows of 128-row block b quantised
    int32_t qg_rows;       // rows per chunk (rows x K x 2 <= kQgBufBytes)
    int32_t qg_chunks;     // ceil(M / qg_rows)
    uint32_t* sk_flag;   // stream-K: [units + 1][2 CTAs][8 epilogue warps] (zero between launches)
    float* sk_partial_head;  // stream-K: the heads' partials, laid out as the tails' in sk_partial
    float* sk_partial;   // stream-K: [units][2 CTAs][8 epilogue warps][32 rows][128 columns];
                         // split-K: [tiles][split_k][4 quarters][epilogue warps / 4 column parts]
                         //          [128 / (epilogue warps / 4) / 4 float4][32 rows]
};

// Stream-K / split-K workspace for `units` CTA pairs: a flag area, then the
// partials. The flag area holds the stream-K marks ((units + 1) x 16 words,
// indexed by the unit whose first segment ends a split tile), then the
// split-K arrival counters (one per tile: a split launch has at most one tile
// per pair; followed by `units` spare words), then the fused linear's
// counters (2 + kQgMaxRowBlocks words). Every region starts zeroed by
// fp8_linear_set_workspace; stream-K flags and all counters return to zero at
// the end of every launch, so one workspace serves any sequence of
// stream-ordered launches of any schedule.
constexpr size_t kSkFlagBytesPerUnit = 2 * 8 * sizeof(uint32_t);
inline size_t sk_flag_words(int units) { return (size_t)(units + 1) * 16; }
inline size_t split_flag_offset_words(int units) { return sk_flag_words(units); }
// Fused linear: rows are quantised in chunks staged in shared memory, one
// staging buffer of kQgBufBytes per quantising warp (kQgBufs of them);
// readiness is counted per 128-row block, so M <= 128 x kQgMaxRowBlocks;
// rows up to kQgMaxK elements (one row must fit a buffer).
constexpr int kQgBufs = 8;
constexpr uint32_t kQgBufBytes = 24576;
constexpr int kQgClaim = 4;  // chunks claimed per atomic (even, >= 2)
constexpr int kQgMaxRowBlocks = 8192;
constexpr int kQgMaxK = 8192;
inline size_t qg_offset_words(int units) { return split_flag_offset_words(units) + 2 * (size_t)units; }
constexpr size_t kSkPartialBytesPerUnit = 2 * 8 * 32 * 128 * sizeof(float);
constexpr int64_t kSkMinKBlocks = 8;  // shorter tiles gain less from a split than it costs
// Split-K pays where a single-CTA tile's k-loop, which at small M is bound by
// the ring's turnover (~1.7 us per 6 k-blocks on B200), is much longer than
// the split's fixed cost (~3.5 us: partial stores, the arrival handshake
// across the GPU, the reduction). Measured: K = 8192 (64 k-blocks) runs 2.1x
// faster at M <= 26 and 1.55x at M = 128; K = 2048 gains nothing.
constexpr int kSplitMinKBlocksTotal = 48;  // split-K: k-blocks of the layer, at least (FP8, 128 per block)
constexpr int kSplitMinKBlocksTotalW8 = 32;  // the same for weight-only (64 bf16 per block: ~13 us plain)
constexpr int kSplitMinKBlocks = 6;        // split-K: k-blocks per piece (one ring), at least
constexpr int kSplitMaxPieces = 8;         // split-K: pieces per tile, at most
constexpr size_t kSplitPieceBytes = 128 * 128 * sizeof(float);  // one fp32 128 x 128 partial
inline size_t sk_flag_area_bytes(int units) {
    return ((qg_offset_words(units) + 2 + kQgMaxRowBlocks) * sizeof(uint32_t) + 4095) & ~(size_t)4095;
}
// The flag area, then two partial areas of `units` x kSkPartialBytesPerUnit:
// stream-K tails' partials (also split-K's), then stream-K heads' partials.
inline size_t stream_k_workspace_bytes(int units) {
    return sk_flag_area_bytes(units) + 2 * (size_t)units * kSkPartialBytesPerUnit;
}

// Tile configurations the plan chooses from.
enum GemmConfig : int32_t {
    kCfgPair256 = 0,    // FP8 x FP8: 256 x 256 tile on a 2-CTA pair (cta_group::2)
    kCfg128x256 = 1,    // FP8 x FP8: 128 x 256 tile on one CTA
    kCfg128x128 = 2,    // FP8 x FP8: 128 x 128 tile on one CTA
    kCfgW8Pair256 = 3,  // bf16 x FP8 weight (weight-only): 256 x 256 tile on a 2-CTA pair
    kCfgW8128x128 = 4,  // bf16 x FP8 weight (weight-only): 128 x 128 tile on one CTA
    kCfgQGPair256 = 5,  // fused linear (bf16 A quantised by the launch, then FP8 x FP8): 256 x 256 pair tile
    kCfgQG128x128 = 6,  // fused linear: 128 x 128 tile on one CTA
    kCfg128x64 = 7,     // FP8 x FP8: 128 x 64 tile on one CTA (few rows: deeper ring, more CTAs)
    kNumCfgs = 8,
};
int gemm_block_m(int cfg);
int gemm_block_n(int cfg);
int gemm_b_box_rows(int cfg);
int gemm_cta_group(int cfg);
bool gemm_weight_only(int cfg);
bool gemm_quantizes_a(int cfg);  // fused linear: bf16 A quantised by the launch before its GEMM
int gemm_k_elems(int cfg);  // K elements per pipeline stage
constexpr int kGemmBlockK = 128;  // bytes = FP8 elements per k-block (one 128 B swizzle row)
constexpr int kGemmStoreBox = 32;

cudaError_t launch_gemm(int cfg, const GemmArgs& args, int units, cudaStream_t stream);
int gemm_units_for(int cfg, int num_tiles, const DeviceInfo* dev);

// Launch `kernel` on `stream` with programmatic stream serialisation allowed
// (and a cluster of `cluster_x` CTAs when > 1).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       int cluster_x, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    int n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (cluster_x > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster_x;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// ------------------------------------------------------------ device side
#if defined(__CUDACC__)

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbarrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Wait for the phase of `bar` with parity `parity` to complete. Gives up when
// *abort becomes non-zero (another role gave up) or after limit_ns; on its own
// expiry it raises *abort and the device error word. Returns true on success.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort,
                                                  const DevErr& err) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (abort != nullptr && *abort) return false;
        if (globaltimer_ns() - t0 > err.limit_ns) {
            if (abort != nullptr) *abort = 1;
            atomicOr(err.word, kDevErrTimeout);
            return false;
        }
    }
}

// TMA 2-D tiled load into shared memory, completion counted on `bar`.
// Coordinates: x = inner (bytes for u8 tensors), y = row. No multicast.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int32_t x,
                                            int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            smem_u32(smem_dst)),
        "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// Untiled bulk copy of `bytes` (a multiple of 16; both addresses 16-byte
// aligned) from global to this CTA's shared memory, completion counted on
// `bar`. No multicast.
__device__ __forceinline__ void bulk_load_g2s(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(smem_dst)),
                 "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
// Hint: bring `bytes` (a multiple of 16; address 16-byte aligned) of global
// memory into L2. No data reaches the SM and nothing waits for it.
__device__ __forceinline__ void prefetch_l2_bulk(const void* gsrc, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(gsrc), "r"(bytes) : "memory");
}
// Order global-memory accesses of the generic proxy (other threads' stores
// this thread has acquired) before this thread's later async-proxy accesses.
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// ---- programmatic dependent launch: a kernel launched with the PDL attribute
// may start while its predecessor in the stream finishes; it must not touch
// global memory the predecessor may write or read before pdl_wait() returns
// (which waits for the predecessor's completion and memory flush).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Let the successor in the stream start launching (its own pdl_wait still
// waits for this kernel to complete).
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---- clusters (2-CTA MMA pairs)
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Address of the same shared-memory location in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t smem_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void st_shared_cluster_u32(uint32_t cluster_addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}

// TMA load for a 2-CTA MMA pair: data lands in this CTA's shared memory, the
// byte count is signalled on `mbar_cluster_addr`, which may be the leader
// CTA's barrier. No multicast.
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map, uint32_t mbar_cluster_addr,
                                                 int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            smem_u32(smem_dst)),
        "l"(map), "r"(mbar_cluster_addr), "r"(x), "r"(y)
        : "memory");
}

// TMA store of a shared-memory box to global memory (bulk-group completion).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* smem_src, int32_t x, int32_t y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(map),
                 "r"(smem_u32(smem_src)), "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait_group() {
    asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}
// Order this thread's generic-proxy shared-memory writes before later async-proxy (TMA) reads.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void named_barrier_sync(uint32_t id, uint32_t threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// ---- tcgen05 with two CTAs per MMA (cta_group::2): issued by the pair's leader.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* smem_slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_slot)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void mma_f8f6f4_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T, bf16 x bf16 -> fp32 (kind::f16).
__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` in every CTA of `cta_mask` when this thread's prior pair MMAs complete.
__device__ __forceinline__ void mma_commit_pair_multicast(uint64_t* bar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"(cta_mask)
        : "memory");
}
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// ---- tcgen05 (one CTA per MMA: cta_group::1)
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_slot)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, E4M3 x E4M3 -> fp32.
__device__ __forceinline__ void mma_f8f6f4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 x bf16 -> fp32 (kind::f16), one CTA.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` when every tcgen05.mma issued so far by this thread has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// 32 lanes x 32 consecutive 32-bit TMEM columns -> 32 registers per thread.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 32 lanes x 16 consecutive 32-bit TMEM columns -> 16 registers per thread.
// The registers are written asynchronously: read them only after
// tmem_wait_ld16() on the same array, which ties their later uses to the wait.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}
// Wait for every tcgen05.ld this thread issued; r's values are valid after it.
__device__ __forceinline__ void tmem_wait_ld16(uint32_t (&r)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15])
                 :
                 : "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile stored the way
// a 128-byte-swizzled TMA load leaves it: rows of 128 B, 8-row (1024 B)
// swizzle atoms stacked along M/N. Fields (sm_100 UMMA descriptor): start
// address >> 4 in bits 0-13, leading byte offset >> 4 in 16-29 (unused for
// swizzled K-major, set to 1), stride byte offset >> 4 in 32-45 (1024 B
// between 8-row groups), version 1 in bits 46-47, swizzle mode in 61-63
// (2 = 128 B).
__device__ __forceinline__ uint64_t umma_desc_kmajor_sw128(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

// Instruction descriptor of kind::f8f6f4, E4M3 x E4M3 -> F32, both K-major.
// Bits: D format 4-5 (1 = F32), A format 7-9 (0 = E4M3), B format 10-12,
// A / B major 15 / 16 (0 = K), N >> 3 in 17-22, M >> 4 in 24-28.
__host__ __device__ constexpr uint32_t umma_idesc_e4m3_f32(int M, int N) {
    return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Instruction descriptor of kind::f16 with BF16 A and B (format 1 in bits 7-9
// and 10-12), F32 accumulator, both K-major.
__host__ __device__ constexpr uint32_t umma_idesc_bf16_f32(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

#endif  // __CUDACC__

}  // namespace fp8dit
