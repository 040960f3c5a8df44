/*
 * The library driven from plain C through include/fp8dit.h alone: no PyTorch,
 * only the CUDA runtime for device memory. Used by tests/test_gpu_c_abi.py.
 *
 * usage: c_abi_harness DIR M N K
 *   reads  DIR/a.bin (bf16 [M, K]), DIR/w.bin (bf16 [N, K]), DIR/bias.bin (bf16 [N])
 *   writes DIR/qw.bin, DIR/sw.bin (per-channel weight codes and scales),
 *          DIR/qa.bin, DIR/sa.bin (per-token activation codes and scales),
 *          DIR/y.bin (bf16 [M, N])
 * Exit status 0 on success; otherwise a message on stderr.
 */
#include <cuda_runtime.h>
#include <stdio.h>
#include <stdlib.h>

#include "fp8dit.h"

static int fail(const char* what) {
    fprintf(stderr, "%s: %s\n", what, fp8dit_last_error_string());
    return 1;
}

static int read_file(const char* dir, const char* name, void* buf, size_t bytes) {
    char path[1024];
    snprintf(path, sizeof(path), "%s/%s", dir, name);
    FILE* f = fopen(path, "rb");
    if (!f) return 0;
    size_t got = fread(buf, 1, bytes, f);
    fclose(f);
    return got == bytes;
}

static int write_file(const char* dir, const char* name, const void* buf, size_t bytes) {
    char path[1024];
    snprintf(path, sizeof(path), "%s/%s", dir, name);
    FILE* f = fopen(path, "wb");
    if (!f) return 0;
    size_t put = fwrite(buf, 1, bytes, f);
    fclose(f);
    return put == bytes;
}

int main(int argc, char** argv) {
    if (argc != 5) {
        fprintf(stderr, "usage: %s DIR M N K\n", argv[0]);
        return 2;
    }
    const char* dir = argv[1];
    const int64_t M = atoll(argv[2]), N = atoll(argv[3]), K = atoll(argv[4]);
    const size_t a_bytes = (size_t)M * K * 2, w_bytes = (size_t)N * K * 2, y_bytes = (size_t)M * N * 2;
    uint16_t* a = malloc(a_bytes);
    uint16_t* w = malloc(w_bytes);
    uint16_t* bias = malloc((size_t)N * 2);
    uint16_t* y = malloc(y_bytes);
    uint8_t* qa = malloc((size_t)M * K);
    uint8_t* qw = malloc((size_t)N * K);
    float* sa = malloc((size_t)M * 4);
    float* sw = malloc((size_t)N * 4);
    if (!a || !w || !bias || !y || !qa || !qw || !sa || !sw) return 3;
    if (!read_file(dir, "a.bin", a, a_bytes) || !read_file(dir, "w.bin", w, w_bytes) ||
        !read_file(dir, "bias.bin", bias, (size_t)N * 2)) {
        fprintf(stderr, "cannot read the inputs\n");
        return 3;
    }
    if (cudaSetDevice(0) != cudaSuccess) return 4;
    uint16_t *d_a, *d_w, *d_bias, *d_y;
    uint8_t *d_qa, *d_qw;
    float *d_sa, *d_sw;
    if (cudaMalloc((void**)&d_a, a_bytes) || cudaMalloc((void**)&d_w, w_bytes) ||
        cudaMalloc((void**)&d_bias, (size_t)N * 2) || cudaMalloc((void**)&d_y, y_bytes) ||
        cudaMalloc((void**)&d_qa, (size_t)M * K) || cudaMalloc((void**)&d_qw, (size_t)N * K) ||
        cudaMalloc((void**)&d_sa, (size_t)M * 4) || cudaMalloc((void**)&d_sw, (size_t)N * 4))
        return 4;
    cudaStream_t s;
    if (cudaStreamCreate(&s) != cudaSuccess) return 4;
    cudaMemcpy(d_a, a, a_bytes, cudaMemcpyHostToDevice);
    cudaMemcpy(d_w, w, w_bytes, cudaMemcpyHostToDevice);
    cudaMemcpy(d_bias, bias, (size_t)N * 2, cudaMemcpyHostToDevice);

    if (fp8_quantize_weight_per_channel(d_w, N, K, FP8DIT_E4M3FN, d_qw, d_sw, s) != FP8DIT_OK)
        return fail("fp8_quantize_weight_per_channel");
    fp8dit_linear h = NULL;
    if (fp8_linear_create(N, K, d_qw, d_sw, d_bias, 0, &h) != FP8DIT_OK) return fail("fp8_linear_create");
    if (fp8_scaled_linear(h, M, d_a, NULL, NULL, d_qa, d_sa, d_y, s) != FP8DIT_OK)
        return fail("fp8_scaled_linear");
    if (fp8dit_device_error(s) != FP8DIT_OK) return fail("fp8dit_device_error");
    if (cudaStreamSynchronize(s) != cudaSuccess) return 4;
    /* An argument error must come back as a status and enqueue nothing. */
    if (fp8_scaled_linear(h, -1, d_a, NULL, NULL, d_qa, d_sa, d_y, s) != FP8DIT_ERR_INVALID_ARG) {
        fprintf(stderr, "negative M was not rejected\n");
        return 5;
    }

    cudaMemcpy(y, d_y, y_bytes, cudaMemcpyDeviceToHost);
    cudaMemcpy(qa, d_qa, (size_t)M * K, cudaMemcpyDeviceToHost);
    cudaMemcpy(sa, d_sa, (size_t)M * 4, cudaMemcpyDeviceToHost);
    cudaMemcpy(qw, d_qw, (size_t)N * K, cudaMemcpyDeviceToHost);
    cudaMemcpy(sw, d_sw, (size_t)N * 4, cudaMemcpyDeviceToHost);
    if (fp8_linear_destroy(h) != FP8DIT_OK) return fail("fp8_linear_destroy");
    if (!write_file(dir, "y.bin", y, y_bytes) || !write_file(dir, "qa.bin", qa, (size_t)M * K) ||
        !write_file(dir, "sa.bin", sa, (size_t)M * 4) || !write_file(dir, "qw.bin", qw, (size_t)N * K) ||
        !write_file(dir, "sw.bin", sw, (size_t)N * 4)) {
        fprintf(stderr, "cannot write the outputs\n");
        return 3;
    }
    cudaFree(d_a); cudaFree(d_w); cudaFree(d_bias); cudaFree(d_y);
    cudaFree(d_qa); cudaFree(d_qw); cudaFree(d_sa); cudaFree(d_sw);
    cudaStreamDestroy(s);
    free(a); free(w); free(bias); free(y); free(qa); free(qw); free(sa); free(sw);
    return 0;
}
