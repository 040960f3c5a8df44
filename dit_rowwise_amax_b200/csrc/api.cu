// C-ABI entry points of libfp8dit (declared and documented in include/fp8dit.h):
// argument validation, per-device state, TMA descriptors, the tile plan bound
// at layer creation, and dispatch to the kernels. Nothing here computes on
// the host: every step of the path runs in the CUDA kernels.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "fp8dit_internal.cuh"
#include "linear_handle.cuh"

// Per-device error word raised by expired bounded waits.
__device__ uint32_t g_fp8dit_error_word;

namespace fp8dit {

// ------------------------------------------------------------------ errors
static thread_local char t_last_error[512];

void set_error(const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_last_error, sizeof(t_last_error), fmt, ap);
    va_end(ap);
}

fp8dit_status cuda_fail(cudaError_t e, const char* what) {
    set_error("%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
    return FP8DIT_ERR_CUDA;
}

static fp8dit_status invalid(const char* msg) {
    set_error("invalid argument: %s", msg);
    return FP8DIT_ERR_INVALID_ARG;
}

static fp8dit_status unsupported(const char* msg) {
    set_error("unsupported shape: %s", msg);
    return FP8DIT_ERR_UNSUPPORTED_SHAPE;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------------- devices
constexpr int kMaxDevices = 64;
static DeviceInfo g_dev[kMaxDevices];
static bool g_dev_ready[kMaxDevices];
static std::mutex g_dev_mutex;

const DeviceInfo* device_info() {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        cuda_fail(e, "cudaGetDevice");
        return nullptr;
    }
    if (dev < 0 || dev >= kMaxDevices) {
        set_error("device ordinal %d beyond %d", dev, kMaxDevices);
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (!g_dev_ready[dev]) {
        DeviceInfo info{};
        int major = 0, minor = 0;
        if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&info.num_sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&info.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) !=
                cudaSuccess) {
            cuda_fail(e, "cudaDeviceGetAttribute");
            return nullptr;
        }
        if (major != 10 || minor != 0) {
            set_error("device %d is sm_%d%d; this library is built for sm_100a only", dev, major, minor);
            return nullptr;
        }
        void* word = nullptr;
        if ((e = cudaGetSymbolAddress(&word, g_fp8dit_error_word)) != cudaSuccess) {
            cuda_fail(e, "cudaGetSymbolAddress(error word)");
            return nullptr;
        }
        info.err_word = static_cast<uint32_t*>(word);
        g_dev[dev] = info;
        g_dev_ready[dev] = true;
    }
    return &g_dev[dev];
}

static DevErr dev_err(const DeviceInfo* d) { return DevErr{d->err_word, kDefaultWaitLimitNs}; }

// ------------------------------------------------------------- TMA maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

fp8dit_status encode_tma_2d(CUtensorMap* map, int elem_bytes, const void* base, uint64_t inner, uint64_t outer,
                            uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                            CUtensorMapSwizzle swizzle) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) {
        set_error("cuTensorMapEncodeTiled is not available from the driver");
        return FP8DIT_ERR_CUDA;
    }
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_stride_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estride[2] = {1, 1};
    const CUtensorMapDataType dt = elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16;
    CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("cuTensorMapEncodeTiled failed (CUresult %d) for %llu x %llu", (int)r, (unsigned long long)outer,
                  (unsigned long long)inner);
        return FP8DIT_ERR_CUDA;
    }
    return FP8DIT_OK;
}

// ------------------------------------------------------------- self test
namespace {
__global__ void selftest_wait_kernel(DevErr err) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbarrier_init();
        // Nothing ever arrives: the bounded wait must expire and report.
        mbar_wait_bounded(&bar, 0, nullptr, err);
    }
}
}  // namespace

cudaError_t launch_selftest_wait(cudaStream_t stream, DevErr err) {
    selftest_wait_kernel<<<1, 32, 0, stream>>>(err);
    return cudaGetLastError();
}

}  // namespace fp8dit

using namespace fp8dit;

int64_t fp8dit::linear_k(const fp8dit_linear_s* h) { return h->K; }
int fp8dit::linear_device(const fp8dit_linear_s* h) { return h->device; }

static int64_t tiles_for(const fp8dit_linear_s* h, int64_t M, int n_problems, int cfg) {
    const int64_t bm = gemm_block_m(cfg), bn = gemm_block_n(cfg);
    return ((M + bm - 1) / bm) * ((h->N + bn - 1) / bn) * n_problems;
}

// Tile plan, a function of (M, N, n_problems, SM count) only:
//  - 256 x 256 tiles on CTA pairs when M fills a pair tile and the tiles keep
//    at least half of the pairs busy;
//  - else 128 x 256 tiles on single CTAs when they keep half the SMs busy;
//  - else 128 x 64 tiles when they fit in one wave (small M: the most CTAs,
//    the deepest ring, the shortest epilogue);
//  - else 128 x 128 tiles.
static int choose_cfg(const fp8dit_linear_s* h, int64_t M, int n_problems) {
    const int pairs = h->num_sms / 2;
    if (M >= 256 && tiles_for(h, M, n_problems, kCfgPair256) * 2 >= pairs) return kCfgPair256;
    if (tiles_for(h, M, n_problems, kCfg128x256) * 2 >= h->num_sms) return kCfg128x256;
    // Few tiles: 128 x 64 tiles while they fit in one wave (twice the CTAs,
    // an 8-deep ring and half the epilogue per CTA of a 128 x 128 tile).
    if (tiles_for(h, M, n_problems, kCfg128x64) <= h->num_sms) return kCfg128x64;
    return kCfg128x128;
}

// Weight-only plan: 256 x 256 pair tiles when M fills them and they keep half
// of the pairs busy, else 128 x 128 tiles on single CTAs.
static int choose_cfg_weight_only(const fp8dit_linear_s* h, int64_t M) {
    const int pairs = h->num_sms / 2;
    if (M >= 256 && tiles_for(h, M, 1, kCfgW8Pair256) * 2 >= pairs) return kCfgW8Pair256;
    return kCfgW8128x128;
}

// Fused-linear plan: the same choice between pair tiles and 128 x 128 tiles.
static int choose_cfg_fused(const fp8dit_linear_s* h, int64_t M) {
    const int pairs = h->num_sms / 2;
    if (M >= 256 && tiles_for(h, M, 1, kCfgQGPair256) * 2 >= pairs) return kCfgQGPair256;
    return kCfgQG128x128;
}

// What the fused linear's launch needs besides the GEMM's operands.
struct QgInputs {
    const uint16_t* a;  // bf16 A [M, K]
    uint8_t* qa;        // its codes (the GEMM's A)
    float* sa;          // its scales
};

// Split-K plan for the single-CTA plans of the FP8 linear and of the
// weight-only linear when a workspace is attached: if 128 x 128 tiles fill at
// most half of the SMs and K has at least kSplitMinKBlocksTotal k-blocks
// (kSplitMinKBlocksTotalW8 of 64 elements for weight-only; each threshold is
// a plain k-loop of ~13 us), each tile is cut into S pieces of at
// least kSplitMinKBlocks k-blocks (S <= kSplitMaxPieces, tiles x S <= SMs), so
// every CTA streams a short slice of W instead of one CTA per tile streaming
// all of K. Returns S (1: no split).
static int split_pieces(const fp8dit_linear* hs, int32_t n, int64_t M, int cfg, int num_sms) {
    const bool wo = cfg == kCfgW8128x128;
    if ((cfg != kCfg128x128 && cfg != kCfg128x256 && cfg != kCfg128x64 && !wo) || hs[0]->sk_ws == nullptr || M <= 0)
        return 1;
    int64_t tiles = 0;
    for (int g = 0; g < n; ++g) tiles += ((M + 127) / 128) * ((hs[g]->N + 127) / 128);
    if (tiles <= 0 || tiles * 2 > num_sms) return 1;
    const int64_t ke = wo ? 64 : 128;  // K elements per k-block of the configuration
    const int64_t num_kb = (hs[0]->K + ke - 1) / ke;
    if (num_kb < (wo ? kSplitMinKBlocksTotalW8 : kSplitMinKBlocksTotal)) return 1;
    // Weight-only above 64 rows with fewer than 64 k-blocks: the heavier
    // reduction cancels the gain (measured: M = 128, K = 2048, 16.1 us plain vs
    // 16.4 split).
    if (wo && M > 64 && num_kb < 2 * kSplitMinKBlocksTotalW8) return 1;
    int64_t S = num_sms / tiles;
    if (S > num_kb / kSplitMinKBlocks) S = num_kb / kSplitMinKBlocks;
    if (S > kSplitMaxPieces) S = kSplitMaxPieces;
    return S >= 2 ? (int)S : 1;
}

// Rows of A per TMA load for the FP8 x FP8 plans. With one row tile on a
// single CTA only M rows (rounded up to 8) are loaded: zero-filling the rest
// of a 128-row box slowed 96 CTAs at M = 26 from 7.7 to 10 us per launch.
static int a_box_rows_for(int cfg, int64_t M) {
    return (gemm_cta_group(cfg) == 1 && M < 128) ? (int)((M + 7) / 8 * 8) : 128;
}

// a: FP8 codes [M, K] (qa) for the FP8 x FP8 configurations (the fused
// linear's included: the launch writes them first), bf16 [M, K] for the
// weight-only ones; sa: per-token scales, or NULL (weight-only); qg: the
// fused linear's bf16 activation and outputs.
static fp8dit_status run_gemm(const fp8dit_linear* hs, int32_t n, int64_t M, const void* a, const float* sa,
                              uint16_t* const* ys, cudaStream_t stream, const DeviceInfo* dev, int cfg,
                              const QgInputs* qg = nullptr) {
    const int split = split_pieces(hs, n, M, cfg, dev->num_sms);
    if (split > 1 && !gemm_weight_only(cfg)) cfg = kCfg128x128;
    const int bm = gemm_block_m(cfg);
    const int bn = gemm_block_n(cfg);
    const int ke = gemm_k_elems(cfg);
    const int64_t K = hs[0]->K;
    GemmArgs args;
    memset(&args, 0, sizeof(args));
    // A: FP8 codes (128-byte rows, swizzled, MMA-ready); weight-only: bf16
    // (128-byte rows of 64 elements, swizzled, MMA-ready).
    fp8dit_status st =
        gemm_weight_only(cfg)
            ? encode_tma_2d(&args.tmA, 2, a, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, (uint32_t)ke, 128,
                            CU_TENSOR_MAP_SWIZZLE_128B)
            : encode_tma_2d(&args.tmA, 1, a, (uint64_t)K, (uint64_t)M, (uint64_t)K, (uint32_t)ke,
                            (uint32_t)a_box_rows_for(cfg, M), CU_TENSOR_MAP_SWIZZLE_128B);
    args.a_box_rows = a_box_rows_for(cfg, M);
    if (st != FP8DIT_OK) return st;
    const int64_t tiles_m64 = (M + bm - 1) / bm;
    int64_t tiles64 = 0;
    for (int g = 0; g < n; ++g) tiles64 += tiles_m64 * ((hs[g]->N + bn - 1) / bn);
    if (tiles64 > INT32_MAX) return unsupported("more than 2^31 - 1 output tiles");
    const int tiles_m = (int)tiles_m64;
    int tiles = 0;
    for (int g = 0; g < n; ++g) {
        args.tmB[g] = hs[g]->tmB[cfg];
        st = encode_tma_2d(&args.tmY[g], 2, ys[g], (uint64_t)hs[g]->N, (uint64_t)M, (uint64_t)hs[g]->N * 2,
                           kGemmStoreBox, kGemmStoreBox, CU_TENSOR_MAP_SWIZZLE_64B);
        if (st != FP8DIT_OK) return st;
        GemmProblem& p = args.prob[g];
        p.sw = hs[g]->sw;
        p.bias = hs[g]->bias;
        p.y = ys[g];
        p.N = (int32_t)hs[g]->N;
        p.tiles_n = (int32_t)((hs[g]->N + bn - 1) / bn);
        p.tile_start = tiles;
        tiles += tiles_m * p.tiles_n;
    }
    // Stream-K when the layer has a workspace and a data-parallel FP8 pair-tile
    // launch would keep its units busy for less than 3/4 of its waves (a nearly
    // empty last wave), with at least kSkMinKBlocks k-blocks per tile.
    // Measured on B200: 150 to 152 tiles on 74 pairs (3 waves, 68% busy) run
    // 2-18% faster split, depending on the power state; 128 tiles (2 waves,
    // 86% busy) run 6% slower, since
    // under the power cap the SMs left idle in a data-parallel last wave let
    // the busy ones clock higher, which recovers most of the idle time.
    int units = gemm_units_for(cfg, tiles, dev);
    const int64_t num_kb = (K + ke - 1) / ke;
    if (split > 1) {
        // One CTA per (tile, piece); tiles * split <= SMs by construction. The
        // arrival counters (one per tile, tiles <= SMs / 2) sit in the flag
        // area after the stream-K flags, the partials in the partial area
        // (tiles * split * 64 KB <= SMs * 64 KB, within (SMs / 2) * 256 KB).
        const int pairs = hs[0]->num_sms / 2;
        units = tiles * split;
        if (units > dev->num_sms || (size_t)units * kSplitPieceBytes > (size_t)pairs * kSkPartialBytesPerUnit ||
            tiles > pairs)
            return unsupported("split-K plan exceeds the workspace");
        args.split_k = split;
        args.split_arrive = static_cast<uint32_t*>(hs[0]->sk_ws) + split_flag_offset_words(pairs);
        args.sk_partial = reinterpret_cast<float*>(static_cast<uint8_t*>(hs[0]->sk_ws) + sk_flag_area_bytes(pairs));
    }
    if (n == 1 && cfg == kCfgPair256 && hs[0]->sk_ws != nullptr && tiles >= units && num_kb >= kSkMinKBlocks) {
        const int64_t waves = (tiles + units - 1) / units;
        if ((waves * units - tiles) * 4 > waves * units) {
            // units <= pairs: the layout is the one the workspace was sized for.
            const int pairs = hs[0]->num_sms / 2;
            uint8_t* ws = static_cast<uint8_t*>(hs[0]->sk_ws);
            args.stream_k = 1;
            args.sk_flag = reinterpret_cast<uint32_t*>(ws);
            args.sk_partial = reinterpret_cast<float*>(ws + sk_flag_area_bytes(pairs));
            args.sk_partial_head =
                reinterpret_cast<float*>(ws + sk_flag_area_bytes(pairs) + (size_t)pairs * kSkPartialBytesPerUnit);
        }
    }
    args.sa = sa;
    if (qg != nullptr) {
        // Rows per staged chunk: as many bf16 rows as fit one staging buffer.
        const int rows = (int)(kQgBufBytes / ((uint32_t)K * 2u));
        args.qg_a = qg->a;
        args.qg_q = qg->qa;
        args.qg_s = qg->sa;
        args.qg_ctr = static_cast<uint32_t*>(hs[0]->sk_ws) + qg_offset_words(hs[0]->num_sms / 2);
        args.qg_rows = rows;
        args.qg_chunks = (int32_t)((M + rows - 1) / rows);
    }
    args.M = (int32_t)M;
    args.K = (int32_t)hs[0]->K;
    args.G = n;
    args.num_tiles = tiles;
    args.num_kb = (int32_t)num_kb;
    args.err = dev_err(dev);
    cudaError_t e = launch_gemm(cfg, args, units, stream);
    if (e != cudaSuccess) return cuda_fail(e, "FP8 GEMM launch");
    return FP8DIT_OK;
}

// Largest sizes the kernels index with 32-bit tile / row arithmetic.
constexpr int64_t kMaxRows = (int64_t)1 << 30;
constexpr int64_t kMaxK = (int64_t)1 << 20;

extern "C" {

const char* fp8dit_last_error_string(void) { return t_last_error; }

fp8dit_status fp8_quantize_rowwise(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, fp8dit_format fmt,
                                   uint8_t* q, int64_t ldq, float* scale, fp8dit_stream_t stream) {
    t_last_error[0] = 0;
    if (fmt != FP8DIT_E4M3FN && fmt != FP8DIT_E5M2) return invalid("format");
    if (M < 0 || K <= 0) return invalid("M must be >= 0 and K > 0");
    if (K % 16 != 0) return unsupported("K must be a multiple of 16");
    if (ldx < K || ldx % 8 != 0) return invalid("ldx must be >= K and a multiple of 8");
    if (ldq < K || ldq % 16 != 0) return invalid("ldq must be >= K and a multiple of 16");
    if (M > kMaxRows || K > kMaxK) return unsupported("M or K too large");
    if (M == 0) return FP8DIT_OK;
    if (!x || !q || !scale) return invalid("null pointer");
    if (!aligned16(x) || !aligned16(q)) return invalid("x and q must be 16-byte aligned");
    if (reinterpret_cast<uintptr_t>(scale) & 3u) return invalid("scale must be 4-byte aligned");
    const DeviceInfo* dev = device_info();
    if (!dev) return FP8DIT_ERR_CUDA;
    cudaError_t e = launch_quantize_rows(x, M, K, ldx, fmt, q, ldq, scale, (cudaStream_t)stream, dev);
    return e == cudaSuccess ? FP8DIT_OK : cuda_fail(e, "rowwise quantise launch");
}

fp8dit_status fp8_act_quantize_rowwise(const uint16_t* h, int64_t M, int64_t K, int64_t ldh,
                                       fp8dit_activation act, uint8_t* q, int64_t ldq, float* scale,
                                       uint16_t* gout, int64_t ldg, fp8dit_stream_t stream) {
    t_last_error[0] = 0;
    if (act != FP8DIT_ACT_GELU_ERF && act != FP8DIT_ACT_GELU_TANH && act != FP8DIT_ACT_SILU)
        return invalid("activation");
    if (M < 0 || K <= 0) return invalid("M must be >= 0 and K > 0");
    if (K % 16 != 0) return unsupported("K must be a multiple of 16");
    if (ldh < K || ldh % 8 != 0) return invalid("ldh must be >= K and a multiple of 8");
    if (ldq < K || ldq % 16 != 0) return invalid("ldq must be >= K and a multiple of 16");
    if (gout && (ldg < K || ldg % 8 != 0)) return invalid("ldg must be >= K and a multiple of 8");
    if (M > kMaxRows || K > kMaxK) return unsupported("M or K too large");
    if (M == 0) return FP8DIT_OK;
    if (!h || !q || !scale) return invalid("null pointer");
    if (!aligned16(h) || !aligned16(q) || (gout && !aligned16(gout))) return invalid("h, q and gout must be 16-byte aligned");
    if (reinterpret_cast<uintptr_t>(scale) & 3u) return invalid("scale must be 4-byte aligned");
    const DeviceInfo* dev = device_info();
    if (!dev) return FP8DIT_ERR_CUDA;
    cudaError_t e = launch_act_quantize_rows(h, M, K, ldh, act, q, ldq, scale, gout, ldg, (cudaStream_t)stream, dev);
    return e == cudaSuccess ? FP8DIT_OK : cuda_fail(e, "activation quantise launch");
}

fp8dit_status fp8_quantize_weight_per_channel(const uint16_t* w, int64_t N, int64_t K, fp8dit_format fmt,
                                              uint8_t* qw, float* sw, fp8dit_stream_t stream) {
    t_last_error[0] = 0;
    if (N <= 0) return invalid("N must be > 0");
    return fp8_quantize_rowwise(w, N, K, K, fmt, qw, K, sw, stream);
}

size_t fp8_quantize_weight_per_tensor_workspace_size(int32_t n_tensors) {
    return per_tensor_workspace_bytes(n_tensors);
}

fp8dit_status fp8_quantize_weight_per_tensor(const fp8dit_tensor_desc* tensors, int32_t n_tensors,
                                             fp8dit_format fmt, void* workspace, size_t ws_bytes,
                                             fp8dit_stream_t stream) {
    t_last_error[0] = 0;
    if (n_tensors < 0) return invalid("n_tensors must be >= 0");
    if (n_tensors == 0 || tensors == nullptr) {
        set_error("invalid input: no tensors to convert");
        return FP8DIT_ERR_EMPTY;
    }
    if (fmt != FP8DIT_E4M3FN && fmt != FP8DIT_E5M2) return invalid("format");
    int64_t total = 0;
    for (int32_t i = 0; i < n_tensors; ++i) {
        const fp8dit_tensor_desc& d = tensors[i];
        if (d.numel < 0) return invalid("numel must be >= 0");
        if (d.src_dtype != FP8DIT_SRC_BF16 && d.src_dtype != FP8DIT_SRC_F16 && d.src_dtype != FP8DIT_SRC_F32)
            return invalid("src_dtype must be FP8DIT_SRC_BF16, FP8DIT_SRC_F16 or FP8DIT_SRC_F32");
        if (d.reserved != 0) return invalid("reserved must be 0");
        if (d.numel == 0) continue;
        if (d.numel > ((int64_t)1 << 40)) return unsupported("tensor too large");
        if (!d.src || !d.dst || !d.scale) return invalid("null pointer in tensor descriptor");
        if (!aligned16(d.src) || !aligned16(d.dst)) return invalid("src and dst must be 16-byte aligned");
        if (reinterpret_cast<uintptr_t>(d.scale) & 3u) return invalid("scale must be 4-byte aligned");
        total += d.numel;
    }
    if (total == 0) {
        set_error("no tensor converted to %s: every tensor is empty", fmt == FP8DIT_E4M3FN ? "float8_e4m3fn"
                                                                                             : "float8_e5m2");
        return FP8DIT_ERR_EMPTY;
    }
    if (!workspace || !aligned16(workspace)) return invalid("workspace must be non-null and 16-byte aligned");
    if (ws_bytes < per_tensor_workspace_bytes(n_tensors)) return invalid("workspace too small");
    const DeviceInfo* dev = device_info();
    if (!dev) return FP8DIT_ERR_CUDA;
    cudaError_t e = launch_per_tensor(tensors, n_tensors, fmt, workspace, (cudaStream_t)stream, dev, dev_err(dev));
    return e == cudaSuccess ? FP8DIT_OK : cuda_fail(e, "per-tensor conversion launch");
}

fp8dit_status fp8_linear_create(int64_t N, int64_t K, const uint8_t* qw, const float* sw, const uint16_t* bias,
                                int device, fp8dit_linear* out) {
    t_last_error[0] = 0;
    if (!out) return invalid("out is null");
    *out = nullptr;
    if (N <= 0 || K <= 0) return invalid("N and K must be > 0");
    if (N % 8 != 0) return unsupported("N must be a multiple of 8");
    if (K % 16 != 0) return unsupported("K must be a multiple of 16");
    if (N > kMaxRows || K > kMaxK) return unsupported("N or K too large");
    if (!qw || !sw) return invalid("qw and sw must be non-null");
    if (!aligned16(qw) || !aligned16(sw)) return invalid("qw and sw must be 16-byte aligned");
    if (bias && !aligned16(bias)) return invalid("bias must be 16-byte aligned");
    int prev = 0;
    cudaError_t e = cudaGetDevice(&prev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (device != prev && (e = cudaSetDevice(device)) != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
    fp8dit_status st = FP8DIT_OK;
    fp8dit_linear_s* h = nullptr;
    const DeviceInfo* dev = device_info();
    if (!dev) {
        st = FP8DIT_ERR_CUDA;
    } else {
        h = new fp8dit_linear_s();
        h->N = N;
        h->K = K;
        h->qw = qw;
        h->sw = sw;
        h->bias = bias;
        h->device = device;
        h->num_sms = dev->num_sms;
        for (int cfg = 0; cfg < kNumCfgs && st == FP8DIT_OK; ++cfg) {
            // FP8 x FP8: 128-byte rows, 128-byte swizzle (MMA-ready). Weight-only:
            // 64-byte rows of codes, unswizzled, decoded to bf16 in shared memory.
            const bool wo = gemm_weight_only(cfg);
            st = encode_tma_2d(&h->tmB[cfg], 1, qw, (uint64_t)K, (uint64_t)N, (uint64_t)K, (uint32_t)gemm_k_elems(cfg),
                               (uint32_t)gemm_b_box_rows(cfg),
                               wo ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B);
        }
    }
    if (device != prev) cudaSetDevice(prev);
    if (st != FP8DIT_OK) {
        delete h;
        return st;
    }
    *out = h;
    return FP8DIT_OK;
}

size_t fp8_linear_workspace_size(fp8dit_linear h) {
    t_last_error[0] = 0;
    if (!h) return 0;
    return stream_k_workspace_bytes(h->num_sms / 2);
}

size_t fp8_linear_workspace_flag_bytes(fp8dit_linear h) {
    t_last_error[0] = 0;
    if (!h) return 0;
    return sk_flag_area_bytes(h->num_sms / 2);
}

fp8dit_status fp8_linear_set_workspace(fp8dit_linear h, void* workspace, size_t bytes) {
    t_last_error[0] = 0;
    if (!h) return invalid("null handle");
    if (workspace == nullptr) {
        h->sk_ws = nullptr;
        h->sk_ws_bytes = 0;
        return FP8DIT_OK;
    }
    const size_t need = stream_k_workspace_bytes(h->num_sms / 2);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return invalid("workspace must be 256-byte aligned");
    if (bytes < need) return invalid("workspace smaller than fp8_linear_workspace_size()");
    int prev = 0;
    cudaError_t e = cudaGetDevice(&prev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (h->device != prev && (e = cudaSetDevice(h->device)) != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
    e = cudaMemset(workspace, 0, sk_flag_area_bytes(h->num_sms / 2));  // the flags and counters
    if (h->device != prev) cudaSetDevice(prev);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the workspace flags");
    h->sk_ws = workspace;
    h->sk_ws_bytes = bytes;
    return FP8DIT_OK;
}

fp8dit_status fp8_linear_destroy(fp8dit_linear h) {
    t_last_error[0] = 0;
    if (h) host_pipe_release(h->pipe);
    delete h;
    return FP8DIT_OK;
}

static fp8dit_status check_device(const fp8dit_linear_s* h) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev != h->device) return invalid("current device differs from the layer's device");
    return FP8DIT_OK;
}

fp8dit_status fp8_scaled_linear(fp8dit_linear h, int64_t M, const uint16_t* a_bf16, const uint8_t* qa,
                                const float* sa, uint8_t* qa_scratch, float* sa_scratch, uint16_t* y,
                                fp8dit_stream_t stream) {
    t_last_error[0] = 0;
    if (!h) return invalid("null handle");
    if (M < 0) return invalid("M must be >= 0");
    if (M > kMaxRows) return unsupported("M too large");
    if (M == 0) return FP8DIT_OK;
    if (!y || !aligned16(y)) return invalid("y must be non-null and 16-byte aligned");
    if (a_bf16) {
        if (qa || sa) return invalid("pass either a_bf16 or (qa, sa), not both");
        if (!qa_scratch || !sa_scratch) return invalid("a_bf16 needs qa_scratch and sa_scratch");
        if (!aligned16(a_bf16) || !aligned16(qa_scratch)) return invalid("a_bf16 and qa_scratch must be 16-byte aligned");
        if (reinterpret_cast<uintptr_t>(sa_scratch) & 3u) return invalid("sa_scratch must be 4-byte aligned");
    } else {
        if (!qa || !sa) return invalid("pass a_bf16, or both qa and sa");
        if (!aligned16(qa)) return invalid("qa must be 16-byte aligned");
        if (reinterpret_cast<uintptr_t>(sa) & 3u) return invalid("sa must be 4-byte aligned");
    }
    fp8dit_status st = check_device(h);
    if (st != FP8DIT_OK) return st;
    const DeviceInfo* dev = device_info();
    if (!dev) return FP8DIT_ERR_CUDA;
    if (a_bf16) {
        cudaError_t e = launch_quantize_rows(a_bf16, M, h->K, h->K, FP8DIT_E4M3FN, qa_scratch, h->K, sa_scratch,
                                             (cudaStream_t)stream, dev);
        if (e != cudaSuccess) return cuda_fail(e, "activation quantise launch");
        qa = qa_scratch;
        sa = sa_scratch;
    }
    return run_gemm(&h, 1, M, qa, sa, &y, (cudaStream_t)stream, dev, choose_cfg(h, M, 1));
}

fp8dit_status fp8_weight_only_linear(fp8dit_linear h, int64_t M, const uint16_t* a_bf16, uint16_t* y,
                                     fp8dit_stream_t stream) {
    t_last_error[0] = 0;
    if (!h) return invalid("null handle");
    if (M < 0) return invalid("M must be >= 0");
    if (M > kMaxRows) return unsupported("M too large");
    if (M == 0) return FP8DIT_OK;
    if (!a_bf16 || !aligned16(a_bf16)) return invalid("a_bf16 must be non-null and 16-byte aligned");
    if (!y || !aligned16(y)) return invalid("y must be non-null and 16-byte aligned");
    fp8dit_status st = check_device(h);
    if (st != FP8DIT_OK) return st;
    const DeviceInfo* dev = device_info();
    if (!dev) return FP8DIT_ERR_CUDA;
    return run_gemm(&h, 1, M, a_bf16, nullptr, &y, (cudaStream_t)stream, dev, choose_cfg_weight_only(h, M));
}

fp8dit_status fp8_scaled_linear_fused(fp8dit_linear h, int64_t M, const uint16_t* a_bf16, uint8_t* qa_scratch,
                                      float* sa_scratch, uint16_t* y, fp8dit_stream_t stream) {
    t_last_error[0] = 0;
    if (!h) return invalid("null handle");
    if (M < 0) return invalid("M must be >= 0");
    if (M > (int64_t)kQgMaxRowBlocks * 128) return unsupported("the fused linear takes at most 1048576 rows");
    if (h->K > kQgMaxK) return unsupported("the fused linear takes K <= 8192");
    if (M == 0) return FP8DIT_OK;
    if (!a_bf16 || !aligned16(a_bf16)) return invalid("a_bf16 must be non-null and 16-byte aligned");
    if (!qa_scratch || !aligned16(qa_scratch)) return invalid("qa_scratch must be non-null and 16-byte aligned");
    if (!sa_scratch || ((uintptr_t)sa_scratch & 3u) != 0) return invalid("sa_scratch must be non-null and 4-byte aligned");
    if (!y || !aligned16(y)) return invalid("y must be non-null and 16-byte aligned");
    if (h->sk_ws == nullptr) return invalid("the fused linear needs a workspace (fp8_linear_set_workspace)");
    fp8dit_status st = check_device(h);
    if (st != FP8DIT_OK) return st;
    const DeviceInfo* dev = device_info();
    if (!dev) return FP8DIT_ERR_CUDA;
    const QgInputs qg{a_bf16, qa_scratch, sa_scratch};
    return run_gemm(&h, 1, M, qa_scratch, sa_scratch, &y, (cudaStream_t)stream, dev, choose_cfg_fused(h, M), &qg);
}

fp8dit_status fp8_scaled_linear_multi(const fp8dit_linear* hs, int32_t n, int64_t M, const uint16_t* a_bf16,
                                      uint8_t* qa_scratch, float* sa_scratch, uint16_t* const* ys,
                                      fp8dit_stream_t stream) {
    t_last_error[0] = 0;
    if (!hs || !ys) return invalid("hs and ys must be non-null");
    if (n < 1 || n > kMaxGroups) return invalid("n must be in 1..4");
    for (int32_t i = 0; i < n; ++i) {
        if (!hs[i]) return invalid("null handle");
        if (hs[i]->K != hs[0]->K || hs[i]->device != hs[0]->device) return invalid("handles differ in K or device");
        if (!ys[i] || !aligned16(ys[i])) return invalid("each ys[i] must be non-null and 16-byte aligned");
    }
    if (M < 0) return invalid("M must be >= 0");
    if (M > kMaxRows) return unsupported("M too large");
    if (M == 0) return FP8DIT_OK;
    if (!a_bf16 || !qa_scratch || !sa_scratch) return invalid("a_bf16, qa_scratch and sa_scratch are required");
    if (!aligned16(a_bf16) || !aligned16(qa_scratch)) return invalid("a_bf16 and qa_scratch must be 16-byte aligned");
    if (reinterpret_cast<uintptr_t>(sa_scratch) & 3u) return invalid("sa_scratch must be 4-byte aligned");
    fp8dit_status st = check_device(hs[0]);
    if (st != FP8DIT_OK) return st;
    const DeviceInfo* dev = device_info();
    if (!dev) return FP8DIT_ERR_CUDA;
    cudaError_t e = launch_quantize_rows(a_bf16, M, hs[0]->K, hs[0]->K, FP8DIT_E4M3FN, qa_scratch, hs[0]->K,
                                         sa_scratch, (cudaStream_t)stream, dev);
    if (e != cudaSuccess) return cuda_fail(e, "activation quantise launch");
    return run_gemm(hs, n, M, qa_scratch, sa_scratch, ys, (cudaStream_t)stream, dev, choose_cfg(hs[0], M, n));
}

fp8dit_status fp8_linear_plan(fp8dit_linear h, int64_t M, int32_t n_problems, int32_t* block_m, int32_t* block_n,
                              int32_t* ctas) {
    t_last_error[0] = 0;
    if (!h || M < 0 || n_problems < 1 || n_problems > kMaxGroups) return invalid("plan arguments");
    int cfg = choose_cfg(h, M, n_problems);
    const fp8dit_linear same[kMaxGroups] = {h, h, h, h};
    const int split = split_pieces(same, n_problems, M, cfg, h->num_sms);
    if (split > 1) cfg = kCfg128x128;
    const int64_t tiles = tiles_for(h, M, n_problems, cfg) * split;
    const int64_t max_units = h->num_sms / gemm_cta_group(cfg);
    if (block_m) *block_m = gemm_block_m(cfg);
    if (block_n) *block_n = gemm_block_n(cfg);
    if (ctas) *ctas = (int32_t)((tiles < max_units ? tiles : max_units) * gemm_cta_group(cfg));
    return FP8DIT_OK;
}

fp8dit_status fp8dit_device_error(fp8dit_stream_t stream) {
    t_last_error[0] = 0;
    const DeviceInfo* dev = device_info();
    if (!dev) return FP8DIT_ERR_CUDA;
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    uint32_t word = 0;
    if ((e = cudaMemcpy(&word, dev->err_word, sizeof(word), cudaMemcpyDeviceToHost)) != cudaSuccess)
        return cuda_fail(e, "reading the device error word");
    if (word != 0) {
        if ((e = cudaMemset(dev->err_word, 0, sizeof(word))) != cudaSuccess)
            return cuda_fail(e, "clearing the device error word");
        set_error("a bounded device wait expired (error word 0x%x)", word);
        return FP8DIT_ERR_TIMEOUT;
    }
    return FP8DIT_OK;
}

fp8dit_status fp8dit_selftest_expired_wait(int64_t limit_ns, fp8dit_stream_t stream) {
    t_last_error[0] = 0;
    if (limit_ns < 1000 || limit_ns > 10000000000ll) return invalid("limit_ns must be in 1e3 .. 1e10");
    const DeviceInfo* dev = device_info();
    if (!dev) return FP8DIT_ERR_CUDA;
    cudaError_t e = launch_selftest_wait((cudaStream_t)stream, DevErr{dev->err_word, (unsigned long long)limit_ns});
    return e == cudaSuccess ? FP8DIT_OK : cuda_fail(e, "self-test launch");
}

fp8dit_status fp8dit_selftest_quotient(unsigned long long* mismatch, fp8dit_stream_t stream) {
    t_last_error[0] = 0;
    if (!mismatch || (reinterpret_cast<uintptr_t>(mismatch) & 7u)) return invalid("mismatch must be 8-byte aligned");
    const DeviceInfo* dev = device_info();
    if (!dev) return FP8DIT_ERR_CUDA;
    cudaError_t e = launch_selftest_quotient(mismatch, (cudaStream_t)stream);
    return e == cudaSuccess ? FP8DIT_OK : cuda_fail(e, "quotient self-test launch");
}

}  // extern "C"
