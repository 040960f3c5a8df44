"""fp8_scaled_linear_noalloc: the linear entry point for callers that cannot
allocate device memory (their framework owns the allocator, or they must not
call cudaMalloc / cudaFree mid-step). It keeps the quantised activation in a
fixed array inside the library instead of caller scratch. Its results must
match fp8_scaled_linear's, call after call, and oversized calls must be
refused. This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from conftest import bf16_tensor_to_f64, to_device_bf16

pytestmark = pytest.mark.gpu

fp8 = pytest.importorskip("dit_rowwise_amax_b200")

OK, UNSUPPORTED = 0, 2


def test_noalloc_matches_scaled_linear_on_consecutive_calls():
    L = fp8.load_library()
    N, K = 1024, 2048
    W = synth.normal_bf16("noalloc/W", (N, K), 0.02)
    bias = synth.normal_bf16("noalloc/bias", (N,), 0.1)
    layer = fp8.FP8Linear.from_weight(to_device_bf16(W), to_device_bf16(bias))
    stream = torch.cuda.current_stream().cuda_stream
    for call, M in enumerate((700, 333)):  # two calls in a row, different data and sizes
        A = synth.normal_bf16(f"noalloc/A{call}", (M, K), 1.0, outlier_p=0.01, outlier_factor=20.0)
        a = to_device_bf16(A)
        y_ref = layer.forward(a)  # caller-provided scratch path
        y = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
        assert L.fp8_scaled_linear_noalloc(layer.handle, M, a.data_ptr(), y.data_ptr(), stream) == OK
        torch.cuda.synchronize()
        ok, worst = oracle.tolerance_ok(bf16_tensor_to_f64(y), bf16_tensor_to_f64(y_ref))
        assert ok, f"call {call}: outside tolerance (worst error / bound {worst:.3f})"


def test_noalloc_refuses_oversized_calls():
    L = fp8.load_library()
    N, K = 256, 8192
    W = synth.normal_bf16("noalloc/W2", (N, K), 0.02)
    layer = fp8.FP8Linear.from_weight(to_device_bf16(W))
    M = (8 << 20) // K + 1  # one row more than the activation array holds
    a = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    y = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    assert L.fp8_scaled_linear_noalloc(layer.handle, M, a.data_ptr(), y.data_ptr(), stream) == UNSUPPORTED
    assert b"fp8_scaled_linear_noalloc" in L.fp8dit_last_error_string()
    torch.cuda.synchronize()
    assert bool(torch.all(y == 7.0)), "a refused call wrote its output"
