"""fp8_scaled_linear_noalloc: the FP8 linear for callers that cannot allocate
device memory (a plugin whose host framework owns the device allocator, or
code that must not call cudaMalloc / cudaFree in the middle of a step, since
those calls can synchronise the device and can fail for lack of memory). It
keeps the quantised activation in a fixed array inside the library instead of
caller scratch.

Its results must equal fp8_scaled_linear's with caller scratch bit for bit
(same kernels, same plan, same codes), call after call, and lie within the
oracle's tolerance of the oracle's linear of the oracle's codes; calls at
exactly the array's limits must work and calls beyond them must be refused.

The file name sorts last so that pytest collects these tests after every
other one: if one of them fails, a run that stops at the first failure
(``pytest -x``) has already run the rest of the suite. The tests also pass
when this file runs alone in a fresh process."""
import numpy as np
import pytest
import torch

import oracle
import synth
from conftest import bf16_tensor_to_f64, to_device_bf16

pytestmark = pytest.mark.gpu

fp8 = pytest.importorskip("dit_rowwise_amax_b200")

OK, UNSUPPORTED = 0, 2
MAX_ACT_BYTES = 8 << 20  # FP8DIT_NOALLOC_MAX_ACT_BYTES
MAX_ROWS = 65536         # FP8DIT_NOALLOC_MAX_ROWS


def make_layer(tag, N, K):
    W = synth.normal_bf16(f"noalloc/{tag}/W", (N, K), 0.02)
    bias = synth.normal_bf16(f"noalloc/{tag}/bias", (N,), 0.1)
    layer = fp8.FP8Linear.from_weight(to_device_bf16(W), to_device_bf16(bias))
    qw_o, sw_o = oracle.quantize_rows(W, oracle.E4M3FN)
    assert np.array_equal(layer.qw.cpu().numpy(), qw_o) and np.array_equal(layer.sw.cpu().numpy(), sw_o)
    return layer, qw_o, sw_o, bias


def noalloc(layer, a, M):
    L = fp8.load_library()
    y = torch.full((M, layer.N), 3.0, dtype=torch.bfloat16, device="cuda")
    st = L.fp8_scaled_linear_noalloc(layer.handle, M, a.data_ptr(), y.data_ptr(),
                                     torch.cuda.current_stream().cuda_stream)
    return st, y


def check_call(layer, qw_o, sw_o, bias, A, rows=None):
    """One no-allocation call: bitwise equal to fp8_scaled_linear with caller
    scratch, and within tolerance of the oracle (on `rows` only, if given)."""
    M = A.shape[0]
    a = to_device_bf16(A)
    st, y = noalloc(layer, a, M)
    assert st == OK, fp8.load_library().fp8dit_last_error_string()
    y_ref = layer.forward(a)  # caller-provided scratch
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16)), "differs from fp8_scaled_linear"
    sel = np.arange(M) if rows is None else np.asarray(rows)
    qa_o, sa_o = oracle.quantize_rows(A[sel], oracle.E4M3FN)
    ref = oracle.linear(qa_o, sa_o, qw_o, sw_o, bias)
    ok, worst = oracle.tolerance_ok(bf16_tensor_to_f64(y)[sel], ref)
    assert ok, f"outside tolerance of the oracle (worst error / bound {worst:.3f})"


def test_noalloc_matches_scaled_linear_on_consecutive_calls():
    layer, qw_o, sw_o, bias = make_layer("a", 1024, 2048)
    for call, M in enumerate((700, 333)):  # two calls in a row, different data and sizes
        A = synth.normal_bf16(f"noalloc/A{call}", (M, 2048), 1.0, outlier_p=0.01, outlier_factor=20.0)
        check_call(layer, qw_o, sw_o, bias, A)


def test_noalloc_at_the_byte_limit():
    """M * K = 8 MiB exactly (4096 x 2048): accepted and correct."""
    layer, qw_o, sw_o, bias = make_layer("b", 256, 2048)
    A = synth.normal_bf16("noalloc/limit_bytes", (MAX_ACT_BYTES // 2048, 2048), 1.0)
    rows = np.r_[0:64, 4096 - 64:4096, np.random.default_rng(0).integers(0, 4096, 128)]
    check_call(layer, qw_o, sw_o, bias, A, rows)


def test_noalloc_at_the_row_limit():
    """M = 65536 rows with K = 128 (both limits reached at once)."""
    layer, qw_o, sw_o, bias = make_layer("c", 64, 128)
    A = synth.normal_bf16("noalloc/limit_rows", (MAX_ROWS, 128), 1.0, outlier_p=0.01, outlier_factor=20.0)
    check_call(layer, qw_o, sw_o, bias, A)


@pytest.mark.parametrize("M,K", [((8 << 20) // 8192 + 1, 8192), (MAX_ROWS + 1, 16)])
def test_noalloc_refuses_oversized_calls(M, K):
    """One row beyond the byte limit (K = 8192), and beyond the row limit at a
    K whose bytes would still fit: refused, nothing written."""
    layer = fp8.FP8Linear.from_weight(to_device_bf16(synth.normal_bf16(f"noalloc/W{K}", (256, K), 0.02)))
    a = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    st, y = noalloc(layer, a, M)
    assert st == UNSUPPORTED
    assert b"fp8_scaled_linear_noalloc" in fp8.load_library().fp8dit_last_error_string()
    torch.cuda.synchronize()
    assert bool(torch.all(y == 3.0)), "a refused call wrote its output"
