// FP8 linear from a bf16 activation for callers that cannot allocate device
// memory.
//
// fp8_scaled_linear() quantises the activation into scratch the caller
// passes in (qa_scratch, sa_scratch). Some callers have no way to obtain that
// memory: a plugin whose host framework owns the device allocator and gives
// the plugin none, or code that must not call cudaMalloc / cudaFree at all
// because those calls can synchronise the whole device and can fail for lack
// of memory in the middle of a step. fp8_scaled_linear_noalloc() serves them:
// the quantised activation lives in a fixed array that is part of this
// library's device image, so the call allocates nothing.
//
// Limits and rules (also stated in include/fp8dit.h):
//  - at most FP8DIT_NOALLOC_MAX_ACT_BYTES bytes of FP8 codes (M * K) and
//    FP8DIT_NOALLOC_MAX_ROWS rows (M); larger calls are rejected;
//  - every GPU that loads the library holds the array until the process
//    exits;
//  - every call on a device uses the same array and leaves its codes and
//    scales there; each call rewrites all of what it reads, so nothing needs
//    clearing, but two calls whose work overlaps on the GPU (for example on
//    two streams) race on the array;
//  - the first call on a device looks up the array's device address (once per
//    device, with that device current); make that first call before any
//    stream capture.
#include <mutex>

#include "fp8dit_internal.cuh"

namespace {

constexpr size_t kNoAllocActBytes = FP8DIT_NOALLOC_MAX_ACT_BYTES;
constexpr int64_t kNoAllocMaxRows = FP8DIT_NOALLOC_MAX_ROWS;

// FP8 activation codes (first kNoAllocActBytes bytes), then the fp32 per-token scales.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocActBytes + kNoAllocMaxRows * sizeof(float)];

constexpr int kMaxDevices = 64;
uint8_t* g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mutex;

// Device address of g_noalloc_scratch on the current device. In host code the
// array's name is only a stand-in, never a device address.
fp8dit_status scratch_address(uint8_t** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fp8dit::cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) {
        fp8dit::set_error("device ordinal %d beyond %d", dev, kMaxDevices);
        return FP8DIT_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return fp8dit::cuda_fail(e, "cudaGetSymbolAddress(no-allocation scratch)");
        g_scratch_addr[dev] = static_cast<uint8_t*>(p);
    }
    *out = g_scratch_addr[dev];
    return FP8DIT_OK;
}

}  // namespace

extern "C" fp8dit_status fp8_scaled_linear_noalloc(fp8dit_linear h, int64_t M, const uint16_t* a_bf16, uint16_t* y,
                                                   fp8dit_stream_t stream) {
    fp8dit::set_error("%s", "");
    if (!h) {
        fp8dit::set_error("invalid argument: null handle");
        return FP8DIT_ERR_INVALID_ARG;
    }
    if (M < 0) {
        fp8dit::set_error("invalid argument: M must be >= 0");
        return FP8DIT_ERR_INVALID_ARG;
    }
    const int64_t K = fp8dit::linear_k(h);
    if (M > kNoAllocMaxRows || M * K > (int64_t)kNoAllocActBytes) {
        fp8dit::set_error(
            "unsupported shape: fp8_scaled_linear_noalloc holds at most %lld rows and %lld bytes of FP8 "
            "activation codes; M = %lld, K = %lld needs %lld bytes (use fp8_scaled_linear with caller scratch)",
            (long long)kNoAllocMaxRows, (long long)kNoAllocActBytes, (long long)M, (long long)K,
            (long long)(M * K));
        return FP8DIT_ERR_UNSUPPORTED_SHAPE;
    }
    if (M == 0) return FP8DIT_OK;
    // The array's address is looked up on the current device, so that must be
    // the layer's device (checked before the lookup, which would otherwise
    // load the library's device image, array included, onto another GPU).
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fp8dit::cuda_fail(e, "cudaGetDevice");
    if (dev != fp8dit::linear_device(h)) {
        fp8dit::set_error("invalid argument: current device differs from the layer's device");
        return FP8DIT_ERR_INVALID_ARG;
    }
    uint8_t* scratch = nullptr;
    fp8dit_status st = scratch_address(&scratch);
    if (st != FP8DIT_OK) return st;
    return fp8_scaled_linear(h, M, a_bf16, nullptr, nullptr, scratch,
                             reinterpret_cast<float*>(scratch + kNoAllocActBytes), y, stream);
}
