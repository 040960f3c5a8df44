"""Failure paths on the GPU without faulting it: host-side argument checks
return a status and launch nothing; a bounded device wait that expires sets
the error word, the host reads FP8DIT_ERR_TIMEOUT, and the context stays
usable."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from conftest import to_device_bf16

pytestmark = pytest.mark.gpu

fp8 = pytest.importorskip("dit_rowwise_amax_b200")

OK, INVALID, UNSUPPORTED, EMPTY, CUDA, TIMEOUT = range(6)


def test_expired_wait_reports_timeout_and_context_survives():
    assert fp8.device_error() == OK
    fp8.selftest_expired_wait(2_000_000)  # 2 ms
    assert fp8.device_error() == TIMEOUT
    assert fp8.device_error() == OK  # read clears it
    a = synth.tiny()["A"]
    q, s = fp8.quantize_rowwise(to_device_bf16(a))
    torch.cuda.synchronize()
    qo, so = oracle.quantize_rows(a, oracle.E4M3FN)
    assert np.array_equal(q.cpu().numpy(), qo)


def test_argument_errors_launch_nothing():
    L = fp8.load_library()
    x = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    q = torch.full((4, 64), 7, dtype=torch.uint8, device="cuda")
    s = torch.zeros(4, dtype=torch.float32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert L.fp8_quantize_rowwise(x.data_ptr(), 4, 60, 64, 0, q.data_ptr(), 64, s.data_ptr(), st) == UNSUPPORTED
    assert b"multiple of 16" in L.fp8dit_last_error_string()
    assert L.fp8_quantize_rowwise(x.data_ptr() + 2, 4, 64, 64, 0, q.data_ptr(), 64, s.data_ptr(), st) == INVALID
    assert L.fp8_quantize_rowwise(None, 4, 64, 64, 0, q.data_ptr(), 64, s.data_ptr(), st) == INVALID
    assert L.fp8_quantize_rowwise(x.data_ptr(), 4, 64, 64, 7, q.data_ptr(), 64, s.data_ptr(), st) == INVALID
    assert L.fp8_quantize_rowwise(x.data_ptr(), -1, 64, 64, 0, q.data_ptr(), 64, s.data_ptr(), st) == INVALID
    assert L.fp8_quantize_rowwise(x.data_ptr(), 4, 64, 60, 0, q.data_ptr(), 64, s.data_ptr(), st) == INVALID
    assert L.fp8_quantize_rowwise(x.data_ptr(), 0, 64, 64, 0, None, 64, None, st) == OK
    torch.cuda.synchronize()
    assert bool(torch.all(q == 7)), "a rejected call wrote its output"


def test_linear_create_and_forward_errors():
    L = fp8.load_library()
    qw = torch.zeros((64, 64), dtype=torch.uint8, device="cuda")
    sw = torch.ones(64, dtype=torch.float32, device="cuda")
    h = ctypes.c_void_p()
    assert L.fp8_linear_create(60, 64, qw.data_ptr(), sw.data_ptr(), None, 0, ctypes.byref(h)) == UNSUPPORTED
    assert L.fp8_linear_create(64, 40, qw.data_ptr(), sw.data_ptr(), None, 0, ctypes.byref(h)) == UNSUPPORTED
    assert L.fp8_linear_create(64, 64, qw.data_ptr() + 1, sw.data_ptr(), None, 0, ctypes.byref(h)) == INVALID
    assert L.fp8_linear_create(64, 64, qw.data_ptr(), sw.data_ptr(), None, 0, ctypes.byref(h)) == OK
    st = torch.cuda.current_stream().cuda_stream
    y = torch.zeros((8, 64), dtype=torch.bfloat16, device="cuda")
    a = torch.zeros((8, 64), dtype=torch.bfloat16, device="cuda")
    qa = torch.zeros((8, 64), dtype=torch.uint8, device="cuda")
    sa = torch.zeros(8, dtype=torch.float32, device="cuda")
    # both an activation and a pre-quantised pair
    assert L.fp8_scaled_linear(h, 8, a.data_ptr(), qa.data_ptr(), sa.data_ptr(), None, None, y.data_ptr(), st) == INVALID
    # bf16 path without scratch
    assert L.fp8_scaled_linear(h, 8, a.data_ptr(), None, None, None, None, y.data_ptr(), st) == INVALID
    # neither
    assert L.fp8_scaled_linear(h, 8, None, None, None, None, None, y.data_ptr(), st) == INVALID
    assert L.fp8_scaled_linear(h, 0, None, None, None, None, None, None, st) == OK
    assert L.fp8_linear_destroy(h) == OK


def test_per_tensor_empty_errors():
    L = fp8.load_library()
    assert L.fp8_quantize_weight_per_tensor(None, 0, 0, None, 0, None) == EMPTY


def test_binding_rejects_wrong_outputs_and_scratch():
    """The binding checks caller-supplied outputs and scratch (dtype, shape,
    device) before the library writes through their pointers."""
    a = torch.zeros((8, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        fp8.quantize_rowwise(a, q=torch.empty((8, 32), dtype=torch.uint8, device="cuda"))
    with pytest.raises(ValueError):
        fp8.quantize_rowwise(a, scale=torch.empty((4,), dtype=torch.float32, device="cuda"))
    layer = fp8.FP8Linear.from_weight(torch.zeros((16, 64), dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(ValueError):
        layer.forward(a, y=torch.empty((8, 16), dtype=torch.float32, device="cuda"))
    with pytest.raises(ValueError):
        layer.forward(a, qa_scratch=torch.empty((4, 64), dtype=torch.uint8, device="cuda"))
    with pytest.raises(ValueError):
        layer.forward_weight_only(a, y=torch.empty((8, 8), dtype=torch.bfloat16, device="cuda"))
    other = fp8.FP8Linear.from_weight(torch.zeros((16, 128), dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(ValueError):
        fp8.scaled_linear_multi([layer, other], a)  # K differs
    with pytest.raises(ValueError):
        fp8.scaled_linear_multi([layer], a, ys=[])
    y = layer.forward(a)  # the defaults still work
    torch.cuda.synchronize()
    assert y.shape == (8, 16)
