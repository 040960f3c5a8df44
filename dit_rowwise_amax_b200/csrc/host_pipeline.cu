// FP8 linear from HOST buffers: the activation streams in, the output streams
// out, and the quantise + GEMM of each chunk of rows runs in between.
//
// The linear itself is fp8_scaled_linear from a bf16 activation ("从 BF16 到
// FP8：HunyuanVideo1.5推理优化复盘", section 三.1: per-token quantisation, FP8
// GEMM, scale / bias / bf16 epilogue). What this file adds is the transfer
// schedule around it. The M rows are cut into chunks of chunk_rows; chunk c
// uses workspace slot c mod slots, which holds the chunk's bf16 activation,
// its FP8 codes and scales, and its bf16 output. Per chunk:
//   copy-in stream : wait until the slot's last compute has read its
//                    activation; copy the chunk's rows host -> device;
//   caller's stream: wait for that copy and for the slot's last copy-out;
//                    quantise + GEMM (fp8_scaled_linear);
//   copy-out stream: wait for that compute; copy the output device -> host.
// So host -> device copies of later chunks, the kernels, and device -> host
// copies of earlier chunks overlap, and the two copy directions run together
// on the full-duplex link. The slot events carry across calls, so the next
// call's input copies start as soon as their slots are free, while this
// call's outputs are still streaming out.
#include <mutex>

#include "fp8dit_internal.cuh"
#include "linear_handle.cuh"

namespace fp8dit {

constexpr int kMaxSlots = 8;

struct HostPipe {
    int device = 0;
    int slots = 0;
    int64_t chunk_rows = 0;
    uint8_t* ws = nullptr;  // caller-owned device workspace
    size_t slot_bytes = 0;
    size_t off_qa = 0, off_sa = 0, off_y = 0;  // offsets inside a slot (the activation is at 0)
    cudaStream_t s_in = nullptr, s_out = nullptr;
    cudaEvent_t in_done[kMaxSlots] = {}, comp_done[kMaxSlots] = {}, out_done[kMaxSlots] = {};
    cudaEvent_t call_done = nullptr;
    bool used[kMaxSlots] = {};
    int next = 0;
    std::mutex mu;  // one call at a time per handle
};

static size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }

// Slot layout: bf16 activation [rows, K], FP8 codes [rows, K], fp32 scales
// [rows], bf16 output [rows, N]; each part starts on a 256-byte boundary.
static void slot_layout(int64_t rows, int64_t K, int64_t N, size_t* off_qa, size_t* off_sa, size_t* off_y,
                        size_t* bytes) {
    const size_t a = round256((size_t)rows * K * 2);
    const size_t qa = round256((size_t)rows * K);
    const size_t sa = round256((size_t)rows * 4);
    const size_t y = round256((size_t)rows * N * 2);
    *off_qa = a;
    *off_sa = a + qa;
    *off_y = a + qa + sa;
    *bytes = a + qa + sa + y;
}

void host_pipe_release(HostPipe* p) {
    if (!p) return;
    int prev = 0;
    const bool switched = cudaGetDevice(&prev) == cudaSuccess && prev != p->device &&
                          cudaSetDevice(p->device) == cudaSuccess;
    // Wait for the pipeline's work in flight (the last compute and copy-out
    // of every slot used), so that the workspace is free when this returns.
    for (int s = 0; s < p->slots; ++s) {
        if (!p->used[s]) continue;
        cudaEventSynchronize(p->comp_done[s]);
        cudaEventSynchronize(p->out_done[s]);
    }
    for (int s = 0; s < kMaxSlots; ++s) {
        if (p->in_done[s]) cudaEventDestroy(p->in_done[s]);
        if (p->comp_done[s]) cudaEventDestroy(p->comp_done[s]);
        if (p->out_done[s]) cudaEventDestroy(p->out_done[s]);
    }
    if (p->call_done) cudaEventDestroy(p->call_done);
    if (p->s_in) cudaStreamDestroy(p->s_in);
    if (p->s_out) cudaStreamDestroy(p->s_out);
    if (switched) cudaSetDevice(prev);
    delete p;
}

static fp8dit_status bad(const char* msg) {
    set_error("invalid argument: %s", msg);
    return FP8DIT_ERR_INVALID_ARG;
}

// Creates the pipeline's streams and events on the current device.
static fp8dit_status pipe_init(HostPipe* p) {
    cudaError_t e = cudaStreamCreateWithFlags(&p->s_in, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&p->s_out, cudaStreamNonBlocking);
    for (int s = 0; s < p->slots && e == cudaSuccess; ++s) {
        e = cudaEventCreateWithFlags(&p->in_done[s], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->comp_done[s], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->out_done[s], cudaEventDisableTiming);
    }
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->call_done, cudaEventDisableTiming);
    return e == cudaSuccess ? FP8DIT_OK : cuda_fail(e, "creating the host pipeline's streams and events");
}

}  // namespace fp8dit

using namespace fp8dit;

size_t fp8_linear_host_workspace_size(fp8dit_linear h, int64_t chunk_rows, int32_t slots) {
    if (!h || chunk_rows <= 0 || slots < 2 || slots > kMaxSlots) return 0;
    size_t qa, sa, y, bytes;
    slot_layout(chunk_rows, h->K, h->N, &qa, &sa, &y, &bytes);
    return bytes * (size_t)slots;
}

fp8dit_status fp8_linear_set_host_pipeline(fp8dit_linear h, void* workspace, size_t bytes, int64_t chunk_rows,
                                           int32_t slots) {
    set_error("%s", "");
    if (!h) return bad("null handle");
    if (workspace == nullptr) {  // detach
        host_pipe_release(h->pipe);
        h->pipe = nullptr;
        return FP8DIT_OK;
    }
    if (chunk_rows <= 0) return bad("chunk_rows must be > 0");
    if (slots < 2 || slots > kMaxSlots) return bad("slots must be in 2..8");
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return bad("workspace must be 256-byte aligned");
    if (bytes < fp8_linear_host_workspace_size(h, chunk_rows, slots))
        return bad("workspace smaller than fp8_linear_host_workspace_size()");
    int prev = 0;
    cudaError_t e = cudaGetDevice(&prev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (prev != h->device && (e = cudaSetDevice(h->device)) != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
    HostPipe* p = new HostPipe();
    p->device = h->device;
    p->slots = slots;
    p->chunk_rows = chunk_rows;
    p->ws = static_cast<uint8_t*>(workspace);
    slot_layout(chunk_rows, h->K, h->N, &p->off_qa, &p->off_sa, &p->off_y, &p->slot_bytes);
    fp8dit_status st = pipe_init(p);
    if (prev != h->device) cudaSetDevice(prev);
    if (st != FP8DIT_OK) {
        host_pipe_release(p);
        return st;
    }
    host_pipe_release(h->pipe);
    h->pipe = p;
    return FP8DIT_OK;
}

fp8dit_status fp8_scaled_linear_host(fp8dit_linear h, int64_t M, const uint16_t* a_host, uint16_t* y_host,
                                     fp8dit_stream_t stream) {
    set_error("%s", "");
    if (!h) return bad("null handle");
    if (M < 0) return bad("M must be >= 0");
    if (M == 0) return FP8DIT_OK;
    if (!a_host || !y_host) return bad("a_host and y_host must be non-null");
    HostPipe* p = h->pipe;
    if (!p) return bad("no host pipeline attached (fp8_linear_set_host_pipeline)");
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev != h->device) return bad("current device differs from the layer's device");
    std::lock_guard<std::mutex> lock(p->mu);
    const cudaStream_t cs = (cudaStream_t)stream;
    const int64_t K = h->K, N = h->N;
    for (int64_t r0 = 0; r0 < M; r0 += p->chunk_rows) {
        const int64_t rows = (M - r0 < p->chunk_rows) ? M - r0 : p->chunk_rows;
        const int s = p->next;
        p->next = (s + 1) % p->slots;
        uint8_t* base = p->ws + (size_t)s * p->slot_bytes;
        uint16_t* a_d = reinterpret_cast<uint16_t*>(base);
        uint8_t* qa_d = base + p->off_qa;
        float* sa_d = reinterpret_cast<float*>(base + p->off_sa);
        uint16_t* y_d = reinterpret_cast<uint16_t*>(base + p->off_y);
        // In: the slot's activation is free once its last compute has run.
        if (p->used[s] && (e = cudaStreamWaitEvent(p->s_in, p->comp_done[s], 0)) != cudaSuccess)
            return cuda_fail(e, "host pipeline wait (copy-in)");
        if ((e = cudaMemcpyAsync(a_d, a_host + r0 * K, (size_t)rows * K * 2, cudaMemcpyHostToDevice, p->s_in)) !=
                cudaSuccess ||
            (e = cudaEventRecord(p->in_done[s], p->s_in)) != cudaSuccess)
            return cuda_fail(e, "host pipeline copy-in");
        // Compute: after the copy-in, and after the slot's last copy-out has read y.
        if ((e = cudaStreamWaitEvent(cs, p->in_done[s], 0)) != cudaSuccess ||
            (p->used[s] && (e = cudaStreamWaitEvent(cs, p->out_done[s], 0)) != cudaSuccess))
            return cuda_fail(e, "host pipeline wait (compute)");
        fp8dit_status st = fp8_scaled_linear(h, rows, a_d, nullptr, nullptr, qa_d, sa_d, y_d, stream);
        if (st != FP8DIT_OK) return st;
        if ((e = cudaEventRecord(p->comp_done[s], cs)) != cudaSuccess) return cuda_fail(e, "host pipeline record");
        // Out.
        if ((e = cudaStreamWaitEvent(p->s_out, p->comp_done[s], 0)) != cudaSuccess ||
            (e = cudaMemcpyAsync(y_host + r0 * N, y_d, (size_t)rows * N * 2, cudaMemcpyDeviceToHost, p->s_out)) !=
                cudaSuccess ||
            (e = cudaEventRecord(p->out_done[s], p->s_out)) != cudaSuccess)
            return cuda_fail(e, "host pipeline copy-out");
        p->used[s] = true;
    }
    // The caller's stream passes this call only when every output row is in y_host.
    if ((e = cudaEventRecord(p->call_done, p->s_out)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(cs, p->call_done, 0)) != cudaSuccess)
        return cuda_fail(e, "host pipeline completion");
    return FP8DIT_OK;
}
