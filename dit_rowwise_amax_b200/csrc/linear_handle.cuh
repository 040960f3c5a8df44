// The linear layer handle behind the C-ABI's opaque fp8dit_linear (private
// to the library's sources).
#pragma once

#include "fp8dit_internal.cuh"

namespace fp8dit {
struct HostPipe;                     // host-buffer pipeline state (host_pipeline.cu)
void host_pipe_release(HostPipe* p);  // frees its streams and events; null is a no-op
}  // namespace fp8dit

struct fp8dit_linear_s {
    int64_t N, K;
    const uint8_t* qw;
    const float* sw;
    const uint16_t* bias;
    int device;
    int num_sms;
    CUtensorMap tmB[fp8dit::kNumCfgs];  // weight descriptors, one per tile configuration
    void* sk_ws;                        // caller-owned stream-K workspace (or null)
    size_t sk_ws_bytes;
    fp8dit::HostPipe* pipe;             // host-buffer pipeline (or null)
};
