/*
 * fp8dit — FP8 linear layer of a diffusion / video DiT on B200 (sm_100a).
 *
 * The path (from "从 BF16 到 FP8：HunyuanVideo1.5推理优化复盘", section 三.1):
 *
 *     BF16 activation -> dynamic per-token FP8 quant -> FP8 GEMM
 *                     -> scale / bias / output dtype
 *
 * with weights quantised per output channel ahead of time (section 二),
 * one quantised activation shared by the Q, K and V projections (section
 * 三.4), an entry that takes an already-quantised (fp8, scale) activation
 * (sections 三.3 and 三.5), and the backend / tile choice bound once when a
 * layer is created (section 三.3). The companion step converts whole weight
 * tensors to float8_e4m3fn or float8_e5m2 with one scale each ("Quantize
 * Model to FP8 Format", inputs model_state_dict and fp8_format).
 *
 * Quantisation recipe ("ComfyUI自定义节点开发适配Stable Diffusion 3.5 FP8技术要点",
 * section "FP8：不只是精度减半", steps 1-4), read for FP8:
 *     amax = max |x|                      (over a row, a channel or a tensor)
 *     S    = fp32(amax) / fmax            IEEE fp32 division; S = 1 if amax == 0
 *     q    = RNEsat(fp32(x) / S)          IEEE fp32 division, then round to the
 *                                         nearest FP8 code (ties to even
 *                                         mantissa), |.| > fmax clamps to fmax
 *     x   ~= decode(q) * S                (the stored scale is S)
 * fmax = 448 for E4M3FN, 57344 for E5M2.
 *
 * Conventions for every entry point
 *  - bf16 tensors are passed as uint16_t bit patterns, FP8 tensors as uint8_t
 *    codes (OCP E4M3FN / E5M2), scales as fp32. All tensors are row-major;
 *    "K-major" means the reduction index is the contiguous one.
 *  - Every tensor pointer is a DEVICE pointer on the current device unless a
 *    parameter says "host". The caller owns all memory: inputs, outputs,
 *    scratch and workspace. The library owns only linear handles.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and enqueue work only after every argument has been validated.
 *    An argument error returns a status and enqueues nothing. There is no
 *    fallback path: a shape the kernels cannot take is an error.
 *  - Device-side bounded waits that expire set a per-device error word;
 *    fp8dit_device_error() reads and clears it.
 *  - On any status other than FP8DIT_OK, fp8dit_last_error_string() (per
 *    thread) describes the failure.
 *  - CUDA graphs: the quantisers, the linear entry points (single, multi,
 *    weight-only, fused, stream-K) and the per-tensor conversion only enqueue
 *    kernels (and, per-tensor, a memset), so they can be captured into a
 *    graph and replayed; each replay reads whatever the captured buffers hold
 *    then. Make the first fp8_act_quantize_rowwise call on a device (it builds
 *    its activation tables and synchronises once) and the first
 *    fp8_scaled_linear_noalloc call on a device before capturing.
 *    fp8_scaled_linear_host uses its own copy streams and is not meant for
 *    capture.
 */
#ifndef FP8DIT_H
#define FP8DIT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FP8DIT_OK = 0,
    FP8DIT_ERR_INVALID_ARG = 1,       /* null / misaligned pointer, negative size, bad format */
    FP8DIT_ERR_UNSUPPORTED_SHAPE = 2, /* K % 16 != 0, N % 8 != 0, size beyond the kernels' range */
    FP8DIT_ERR_EMPTY = 3,             /* per-tensor conversion with nothing to convert */
    FP8DIT_ERR_CUDA = 4,              /* a CUDA runtime / driver call failed */
    FP8DIT_ERR_TIMEOUT = 5            /* a bounded device wait expired */
} fp8dit_status;

typedef enum { FP8DIT_E4M3FN = 0, FP8DIT_E5M2 = 1 } fp8dit_format;

/* Same type as cudaStream_t; the header does not need the CUDA headers. */
typedef struct CUstream_st* fp8dit_stream_t;

/* Opaque handle of one FP8 linear layer (see fp8_linear_create). */
typedef struct fp8dit_linear_s* fp8dit_linear;

/*
 * Per-token (rowwise) quantisation of a bf16 activation.
 * ("从 BF16 到 FP8", section 三.1: dynamic per-token FP8 quant; recipe above.)
 *   x     [M, K] bf16, row stride ldx elements (ldx >= K, ldx % 8 == 0), 16-byte aligned.
 *   q     [M, K] FP8 codes of format fmt, row stride ldq bytes (ldq >= K, ldq % 16 == 0),
 *         16-byte aligned.
 *   scale [M] fp32: S of each row.
 * Requires K % 16 == 0 and K > 0, M >= 0 (M == 0 is a no-op). Any K that is a
 * multiple of 16 is accepted. Inputs must be finite.
 */
fp8dit_status fp8_quantize_rowwise(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                                   fp8dit_format fmt, uint8_t* q, int64_t ldq, float* scale,
                                   fp8dit_stream_t stream);

/* Activations a producer kernel can apply before quantising. */
typedef enum {
    FP8DIT_ACT_GELU_ERF = 1,  /* x Phi(x) = x/2 (1 + erf(x / sqrt 2)) */
    FP8DIT_ACT_GELU_TANH = 2, /* x/2 (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))) */
    FP8DIT_ACT_SILU = 3       /* x / (1 + exp(-x)) */
} fp8dit_activation;

/*
 * Producer fusion ("从 BF16 到 FP8", section 三.5): the GELU / SiLU in front of
 * FFN-down emits the (FP8 tensor, per-token scale) pair directly instead of a
 * bf16 tensor that a separate pass then quantises.
 *   h     [M, K] bf16 (the FFN-up output), row stride ldh elements (ldh % 8 == 0), 16-byte aligned.
 *   g     = bf16_rne(act(h)): act evaluated in double (CUDA's double erfc / exp,
 *         every other step an IEEE double operation) and rounded once to bf16,
 *         ties to even; stored to gout [M, K] (row stride ldg, 16-byte aligned)
 *         when gout != NULL.
 *   q, scale: the rowwise recipe applied to g, E4M3FN codes (the GEMM's input).
 * Same shape rules as fp8_quantize_rowwise. The first call on a device builds
 * a 128 KB table per activation (bf16(act(x)) for all 65536 bf16 x, in static
 * device memory) and synchronises `stream` once; make that first call before
 * any stream capture.
 */
fp8dit_status fp8_act_quantize_rowwise(const uint16_t* h, int64_t M, int64_t K, int64_t ldh,
                                       fp8dit_activation act, uint8_t* q, int64_t ldq, float* scale,
                                       uint16_t* gout, int64_t ldg, fp8dit_stream_t stream);

/*
 * Per-output-channel quantisation of a bf16 weight W [N, K] (K contiguous):
 * the rowwise recipe applied to each of the N rows, producing the K-major
 * FP8 weight the GEMM consumes with no transpose ("从 BF16 到 FP8", section
 * 二: parameters quantised per channel ahead of time; section 三.1: B must
 * stay column-major, never transposed and made contiguous).
 *   w [N, K] bf16 contiguous; qw [N, K] codes contiguous; sw [N] fp32.
 * Requires N > 0, K > 0, K % 16 == 0.
 */
fp8dit_status fp8_quantize_weight_per_channel(const uint16_t* w, int64_t N, int64_t K,
                                              fp8dit_format fmt, uint8_t* qw, float* sw,
                                              fp8dit_stream_t stream);

/* Element types a per-tensor conversion reads (a state-dict's floating dtypes). */
typedef enum {
    FP8DIT_SRC_BF16 = 0, /* bfloat16 bit patterns (the default: a zeroed field) */
    FP8DIT_SRC_F16 = 1,  /* IEEE binary16 bit patterns */
    FP8DIT_SRC_F32 = 2   /* IEEE binary32 */
} fp8dit_src_dtype;

/* One tensor of a per-tensor conversion. Pointers are device pointers. */
typedef struct {
    const void* src;   /* numel values of src_dtype, contiguous, 16-byte aligned */
    int64_t numel;     /* >= 0, any size */
    uint8_t* dst;      /* numel FP8 codes, 16-byte aligned */
    float* scale;      /* one fp32: S of the tensor (left untouched when numel == 0) */
    int32_t src_dtype; /* fp8dit_src_dtype of src */
    int32_t reserved;  /* must be 0 */
} fp8dit_tensor_desc;

/* Bytes of device workspace fp8_quantize_weight_per_tensor needs for n tensors. */
size_t fp8_quantize_weight_per_tensor_workspace_size(int32_t n_tensors);

/*
 * Per-tensor conversion of a weight set (a state-dict's tensors) to FP8 with
 * one amax scale per tensor ("Quantize Model to FP8 Format": model_state_dict
 * in, quantised state-dict out in float8_e4m3fn or float8_e5m2). Each tensor
 * may be bf16, fp16 or fp32 (its src_dtype); every value is exact in fp32, so
 * the recipe above applies unchanged: amax = max |x|, S = amax / fmax and
 * q = RNEsat(x / S), both IEEE fp32 divisions.
 *   tensors   HOST array of n_tensors descriptors; it may be freed on return.
 *   workspace DEVICE scratch of at least
 *             fp8_quantize_weight_per_tensor_workspace_size(n_tensors) bytes,
 *             16-byte aligned; its contents on entry do not matter. It must not
 *             be used by another call that runs at the same time on the GPU.
 * Errors: FP8DIT_ERR_EMPTY when n_tensors == 0 or every numel is 0 (the page's
 * "Invalid input." and "No tensor converted to <fp8_format>." outcomes).
 */
fp8dit_status fp8_quantize_weight_per_tensor(const fp8dit_tensor_desc* tensors, int32_t n_tensors,
                                             fp8dit_format fmt, void* workspace, size_t ws_bytes,
                                             fp8dit_stream_t stream);

/*
 * Create an FP8 linear layer y = (A W^T) * sa * sw + bias with E4M3FN
 * operands, fp32 accumulation and bf16 output. The tile plan for every
 * M-bucket and the weight's TMA descriptors are built here, once
 * ("从 BF16 到 FP8", section 三.3: backend chosen from weight shape, device
 * and bias contract at construction, forward does no such checks).
 *   qw   [N, K] E4M3FN codes, K contiguous (from fp8_quantize_weight_per_channel).
 *   sw   [N] fp32 per-channel scales.
 *   bias [N] bf16, or NULL for no bias.
 * The handle BORROWS qw, sw and bias: they must stay valid and unchanged
 * until fp8_linear_destroy. device is the CUDA device that holds them.
 * Requires N % 8 == 0, K % 16 == 0; qw, sw and bias 16-byte aligned.
 */
fp8dit_status fp8_linear_create(int64_t N, int64_t K, const uint8_t* qw, const float* sw,
                                const uint16_t* bias, int device, fp8dit_linear* out);

fp8dit_status fp8_linear_destroy(fp8dit_linear h);

/*
 * Optional stream-K workspace for a layer. When a layer's 256 x 256 output
 * tiles would keep the CTA pairs busy for less than 3/4 of the waves of a
 * tile-per-pair schedule (a nearly empty last wave: e.g. 150 tiles on 74
 * pairs) and a tile has at least 8 k-blocks of 128, each pair instead takes
 * an equal share of the layer's k-blocks; a tile split between two pairs is
 * finished by whichever of the two gets there second, from the fp32 partial
 * the other has stored in this workspace; neither waits for the other, so the
 * launch does not need all of its pairs resident at once. Results stay
 * deterministic (the two parts are added once, in fp32, whichever side
 * finishes) but differ in rounding from the plain schedule.
 * The same workspace enables split-K for few tiles and a long K: when the
 * 128 x 128 tiles of a small-M call fill at most half of the SMs and K has at
 * least 48 k-blocks of 128 (K >= 6144; e.g. text tokens through an FFN-down
 * weight), each tile is cut into up to 8 pieces of at least 6 k-blocks on
 * separate CTAs; every piece stores its fp32 partial and the piece that
 * arrives last adds all of them in piece order for the whole tile
 * (deterministic, rounding differs from the plain schedule). No piece waits
 * for another, so split-K launches need not have all their CTAs resident at
 * once and may share the GPU with other kernels.
 * fp8_weight_only_linear splits the same way from 32 k-blocks of 64 (K >=
 * 2048; K >= 4096 above 64 rows). fp8_scaled_linear_multi uses the workspace
 * of its first layer. Without a workspace, or for other shapes (the
 * FFN shapes among them), the plain schedule is used.
 *   fp8_linear_workspace_size: bytes needed on the layer's device (~38 MB on
 *     148 SMs), the same for every M.
 *   fp8_linear_set_workspace: attach caller-owned DEVICE memory (256-byte
 *     aligned, at least that size) or detach with NULL, while no call that
 *     uses the layer is in flight. Attaching clears the workspace's flags
 *     and counters (synchronously); every launch leaves them cleared, so
 *     stream-ordered launches and replays of a captured CUDA graph need no
 *     host reset. After a call whose device error word reports
 *     FP8DIT_ERR_TIMEOUT, attach the workspace again before reusing it (an
 *     interrupted launch can leave a flag or a count behind). The
 *     workspace may be attached to several layers whose calls run one after
 *     another on the GPU; calls that overlap on the GPU must not share a
 *     workspace.
 */
size_t fp8_linear_workspace_size(fp8dit_linear h);
fp8dit_status fp8_linear_set_workspace(fp8dit_linear h, void* workspace, size_t bytes);
/* Bytes at the start of the workspace that hold its flags and counters: zero
 * after attaching and between launches (the rest holds fp32 partials). */
size_t fp8_linear_workspace_flag_bytes(fp8dit_linear h);

/*
 * Forward of one FP8 linear layer ("从 BF16 到 FP8", sections 三.1, 三.3, 三.5):
 *  - ordinary tensor: a_bf16 != NULL. A [M, K] bf16 (contiguous) is quantised
 *    per token into qa_scratch [M, K] and sa_scratch [M] (both caller-owned,
 *    written by this call), then multiplied. qa and sa must be NULL.
 *  - FP8 tensor: a_bf16 == NULL. qa [M, K] E4M3FN codes (contiguous) and
 *    sa [M] fp32 per-token scales are used as given; the scratch arguments
 *    are ignored.
 *   y [M, N] bf16 contiguous, 16-byte aligned:
 *     y[m, n] = bf16_rne((sum_k dec(qa[m,k]) dec(qw[n,k])) * sa[m] * sw[n] + bias[n])
 * M == 0 is a no-op. Must run on the handle's device.
 */
fp8dit_status fp8_scaled_linear(fp8dit_linear h, int64_t M, const uint16_t* a_bf16,
                                const uint8_t* qa, const float* sa, uint8_t* qa_scratch,
                                float* sa_scratch, uint16_t* y, fp8dit_stream_t stream);

/*
 * FP8 weight-only linear: the FP8 weight-only configuration with scales that
 * the longcat-avatar-compare page sets against NVFP4 W4A4 (section 速度总览). The
 * activation is not quantised; the layer's E4M3 weight is decoded to bf16 in
 * shared memory and multiplied on the BF16 tensor cores:
 *   y[m, n] = bf16_rne( (sum_k A[m,k] dec(qw[n,k])) * sw[n] + bias[n] ), fp32 accumulation.
 *   a_bf16 [M, K] bf16 contiguous, y [M, N] bf16 contiguous, both 16-byte aligned.
 * Uses the same handle (qw, sw, bias) as fp8_scaled_linear.
 */
fp8dit_status fp8_weight_only_linear(fp8dit_linear h, int64_t M, const uint16_t* a_bf16, uint16_t* y,
                                     fp8dit_stream_t stream);

/*
 * The FP8 linear from a bf16 activation in ONE launch (the fused variant of
 * "从 BF16 到 FP8", section 三.1: runtime per-token activation quantisation
 * feeding the FP8 GEMM; section 三.2 item 2: fewer extra reads and writes and
 * intermediate launches). The launch's CTAs first quantise A together: each
 * claims chunks of rows in row order, stages their bf16 values in shared
 * memory with bulk copies, and writes each row's E4M3 codes and scale with
 * the rowwise quantiser's arithmetic; every element is quantised exactly once.
 * Each CTA then runs the FP8 GEMM + epilogue of fp8_scaled_linear, a tile
 * starting as soon as its rows have been quantised. A chunk is only ever
 * claimed by a running CTA and that work waits for nothing, so no wait
 * depends on CTAs that have not started.
 * Result: qa_scratch and sa_scratch hold exactly what fp8_quantize_rowwise
 * writes, and y equals fp8_scaled_linear(h, M, a_bf16, ...) bit for bit where
 * both use 256 x 256 pair tiles (otherwise within the accumulation-order
 * difference of another tile plan).
 *   a_bf16     [M, K] bf16 contiguous, 16-byte aligned;
 *   qa_scratch [M, K] E4M3FN codes, 16-byte aligned, caller-owned: written;
 *   sa_scratch [M] fp32 per-token scales, 4-byte aligned, caller-owned: written;
 *   y          [M, N] bf16 contiguous, 16-byte aligned.
 * The layer must have a workspace attached (fp8_linear_set_workspace): its
 * counters, which every launch leaves at zero; calls that overlap on the GPU
 * must not share it. Requires K <= 8192 and M <= 1048576
 * (FP8DIT_ERR_UNSUPPORTED_SHAPE otherwise). M == 0 is a no-op. Must run on
 * the handle's device.
 */
fp8dit_status fp8_scaled_linear_fused(fp8dit_linear h, int64_t M, const uint16_t* a_bf16, uint8_t* qa_scratch,
                                      float* sa_scratch, uint16_t* y, fp8dit_stream_t stream);

/*
 * FP8 linear from HOST buffers, with the transfers pipelined around the
 * kernels (the library's runtime for callers whose activations live in host
 * memory; the pages have no counterpart). The result is fp8_scaled_linear's
 * from a bf16 activation, row for row (each row depends only on its own
 * activation row), computed chunk by chunk.
 *
 * fp8_linear_host_workspace_size: DEVICE bytes for `slots` slots of
 *   `chunk_rows` rows (per slot: bf16 activation, FP8 codes, scales, bf16
 *   output); 0 for invalid arguments (slots must be 2..8, chunk_rows > 0).
 * fp8_linear_set_host_pipeline: attach caller-owned DEVICE memory (256-byte
 *   aligned, at least that size) to the layer, creating two copy streams and
 *   the slot events on the layer's device; NULL workspace detaches (and frees
 *   the streams and events). Replacing or detaching a pipeline, and
 *   fp8_linear_destroy, first wait on the host for that pipeline's work in
 *   flight. The workspace belongs to this layer only and must stay allocated
 *   until the work of every call using it has completed.
 * fp8_scaled_linear_host: y_host [M, N] = the linear of a_host [M, K] (both
 *   bf16, contiguous, HOST memory; page-locked memory is needed for the
 *   copies to overlap anything). The M rows go in chunks: host-to-device copy
 *   (copy-in stream) -> quantise + GEMM (`stream`) -> device-to-host copy
 *   (copy-out stream), chunks and slots in a ring, so both copy directions and
 *   the kernels overlap, also with the previous call's copy-out.
 *   Ordering: `stream` passes the end of this call only once every output row
 *   is in y_host, so synchronising `stream` (or work queued on it later) sees
 *   the result. The input copies are ordered only after earlier calls' use of
 *   the same slots, NOT after other work queued on `stream`: a_host must hold
 *   the activation when the call is made and stay unchanged, and both host
 *   buffers stay allocated, until `stream` has passed this call. Calls on one
 *   handle are serialised by a lock. Errors as fp8_scaled_linear, plus
 *   FP8DIT_ERR_INVALID_ARG when no pipeline is attached.
 */
size_t fp8_linear_host_workspace_size(fp8dit_linear h, int64_t chunk_rows, int32_t slots);
fp8dit_status fp8_linear_set_host_pipeline(fp8dit_linear h, void* workspace, size_t bytes, int64_t chunk_rows,
                                           int32_t slots);
fp8dit_status fp8_scaled_linear_host(fp8dit_linear h, int64_t M, const uint16_t* a_host, uint16_t* y_host,
                                     fp8dit_stream_t stream);

/*
 * fp8_scaled_linear from a bf16 activation, for callers that cannot allocate
 * device memory. The pages have no counterpart: this entry exists for code
 * that has no way to hand the library qa / sa scratch, such as a plugin whose
 * host framework owns the device allocator, or code that must not call
 * cudaMalloc / cudaFree because they can synchronise the device and can fail
 * for lack of memory mid-step. The quantised activation is kept in a fixed
 * array that is part of the library's device image instead, so this call
 * allocates nothing.
 *   a_bf16 [M, K] bf16 contiguous, y [M, N] bf16 contiguous, both 16-byte
 *   aligned; results equal fp8_scaled_linear(h, M, a_bf16, NULL, NULL, ...).
 * Limits: M <= FP8DIT_NOALLOC_MAX_ROWS and M * K <= FP8DIT_NOALLOC_MAX_ACT_BYTES;
 * larger calls return FP8DIT_ERR_UNSUPPORTED_SHAPE and enqueue nothing.
 * Every GPU that loads the library holds the array (about 8.25 MiB) until the
 * process exits. All calls on a device share it and leave their data in it;
 * each call rewrites everything it reads, but calls whose work overlaps on the
 * GPU (e.g. on two streams) race. The first call on a device looks up the
 * array's device address; make that call before any stream capture.
 */
#define FP8DIT_NOALLOC_MAX_ACT_BYTES (8u << 20)
#define FP8DIT_NOALLOC_MAX_ROWS 65536
fp8dit_status fp8_scaled_linear_noalloc(fp8dit_linear h, int64_t M, const uint16_t* a_bf16, uint16_t* y,
                                        fp8dit_stream_t stream);

/*
 * n linear layers that read the same activation ("从 BF16 到 FP8", section
 * 三.4: quantise hidden_states once and feed the separate Q, K and V
 * projections). A [M, K] bf16 is quantised once into qa_scratch / sa_scratch,
 * then all n products run in one grouped launch.
 *   hs  HOST array of n handles (1 <= n <= 4), all with the same K and device.
 *   ys  HOST array of n device pointers, ys[i] is [M, N_i] bf16.
 * Results are bitwise identical to n fp8_scaled_linear calls whenever the
 * grouped launch and the single calls use the same tile plan and no split
 * (e.g. the 256 x 256 pair plan of the hidden_states projections); a split
 * schedule (workspace attached) may cut the grouped launch's K differently
 * from a single call's and round differently, within the same bound.
 */
fp8dit_status fp8_scaled_linear_multi(const fp8dit_linear* hs, int32_t n, int64_t M,
                                      const uint16_t* a_bf16, uint8_t* qa_scratch,
                                      float* sa_scratch, uint16_t* const* ys,
                                      fp8dit_stream_t stream);

/*
 * Tile plan that fp8_scaled_linear / _multi use for this handle at this M
 * (n_problems = 1 for a single layer): block_m x block_n output tiles,
 * `ctas` thread blocks. For reports and tests.
 */
fp8dit_status fp8_linear_plan(fp8dit_linear h, int64_t M, int32_t n_problems, int32_t* block_m,
                              int32_t* block_n, int32_t* ctas);

/*
 * Synchronise `stream`, then read and clear the current device's error word.
 * Returns FP8DIT_ERR_TIMEOUT if a bounded device wait expired since the last
 * read, FP8DIT_ERR_CUDA if the synchronisation failed, else FP8DIT_OK.
 */
fp8dit_status fp8dit_device_error(fp8dit_stream_t stream);

/*
 * Launch one block whose single thread waits, with the library's bounded
 * wait, on an mbarrier that nothing arrives at, for at most limit_ns
 * nanoseconds (1e3 .. 1e10). The wait expires and sets the error word, so
 * the next fp8dit_device_error() reports FP8DIT_ERR_TIMEOUT. Exercises the
 * failure path without faulting the GPU.
 */
fp8dit_status fp8dit_selftest_expired_wait(int64_t limit_ns, fp8dit_stream_t stream);

/*
 * Exhaustive check of the quantisers' quotient arithmetic: for every finite
 * positive bf16 amax and every bf16 x with |x| <= amax, the FP8 code the
 * quantisers produce for x / S (S = amax / fmax) is compared with the code of
 * the IEEE fp32 division x / S, for E4M3FN and E5M2. Adds the number of
 * differing codes to mismatch[0] (E4M3FN) and mismatch[1] (E5M2), a DEVICE
 * array of two uint64 the caller zeroes. Asynchronous on `stream`.
 */
fp8dit_status fp8dit_selftest_quotient(unsigned long long* mismatch, fp8dit_stream_t stream);

/* Description of the last failure on this thread ("" if none). */
const char* fp8dit_last_error_string(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8DIT_H */
