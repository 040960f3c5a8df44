"""FP8 linear with the per-token quantisation inside the GEMM
(fp8_scaled_linear_fused) on the GPU vs the CPU oracle.

The pre-pass's per-token scales must equal the oracle's bit for bit, and its
reciprocals must be RN(1 / S) where the corrected-reciprocal quotient applies
(amax >= 2^-64) and 0 elsewhere. The output is compared with the oracle's
exact product of the oracle's own codes (|gpu - ref| <= 1e-2 |ref| +
1e-3 rms(ref)), and, where both run 256 x 256 pair tiles, with the unfused
fp8_scaled_linear bit for bit: the in-GEMM codes must be the rowwise
quantiser's."""

import numpy as np
import pytest
import torch

import oracle
import synth
from conftest import bf16_tensor_to_f64, to_device_bf16

pytestmark = pytest.mark.gpu

fp8 = pytest.importorskip("dit_rowwise_amax_b200")


def make_layer(W, bias):
    qw, sw = fp8.quantize_weight_per_channel(to_device_bf16(W))
    layer = fp8.FP8Linear(qw, sw, None if bias is None else to_device_bf16(bias))
    torch.cuda.synchronize()
    return layer, qw.cpu().numpy(), sw.cpu().numpy()


def expected_rcp(A, s):
    """RN(1 / S) in fp32 where amax >= 2^-64, else 0."""
    amax = np.abs(synth.bf16_to_f32(A)).max(axis=1)
    with np.errstate(over="ignore"):  # 1 / S overflows only where the reciprocal is not used
        r = (np.float32(1.0) / s).astype(np.float32)
    return np.where(amax >= np.float32(2.0 ** -64), r, np.float32(0.0)).astype(np.float32)


def run_fused(layer, A):
    M = A.shape[0]
    scratch = torch.empty((2 * M,), dtype=torch.float32, device="cuda")
    y = layer.forward_fused(to_device_bf16(A), scale_scratch=scratch)
    torch.cuda.synchronize()
    assert fp8.device_error() == 0
    qa, sa = oracle.quantize_rows(A, oracle.E4M3FN)
    got = scratch.cpu().numpy()
    assert np.array_equal(got[:M], sa), "per-token scales differ"
    assert np.array_equal(got[M:], expected_rcp(A, sa)), "reciprocals differ"
    return y, qa, sa


def check_rows(y, qa, sa, qw, sw, bias, rows):
    ref = oracle.linear(np.ascontiguousarray(qa[rows]), sa[rows], qw, sw, bias)
    ok, worst = oracle.tolerance_ok(bf16_tensor_to_f64(y)[rows], ref)
    assert ok, f"tolerance exceeded: worst error / bound = {worst:.3f}"


@pytest.mark.parametrize("cfg", ["ffn_up", "ffn_down"])
def test_ffn_full_size_matches_unfused_bitwise(cfg):
    d = getattr(synth, cfg)()
    layer, qw, sw = make_layer(d["W"], d["bias"])
    M = d["A"].shape[0]
    assert layer.plan(M)[:2] == (256, 256)
    y, qa, sa = run_fused(layer, d["A"])
    y_ref = layer.forward(to_device_bf16(d["A"]))
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16)), "fused and unfused outputs differ"
    rng = np.random.default_rng(3)
    rows = np.unique(np.concatenate([np.arange(32), np.arange(M - 32, M), rng.integers(0, M, 32)]))
    check_rows(y, qa, sa, qw, sw, d["bias"], rows)


def test_tiny_config_full():
    d = synth.tiny()
    layer, qw, sw = make_layer(d["W"], d["bias"])
    y, qa, sa = run_fused(layer, d["A"])
    check_rows(y, qa, sa, qw, sw, d["bias"], np.arange(64))


@pytest.mark.parametrize("M", [1, 26, 129, 257, 300])
@pytest.mark.parametrize("N,K", [(8, 16), (136, 48), (520, 2064), (2048, 2048)])
def test_ragged_shapes(M, N, K):
    A = synth.normal_bf16(f"gpu/fused/A/{M}x{K}", (M, K), 1.0, outlier_p=0.01, outlier_factor=20.0)
    W = synth.normal_bf16(f"gpu/fused/W/{N}x{K}", (N, K), 0.02)
    bias = synth.normal_bf16(f"gpu/fused/b/{N}", (N,), 0.1)
    layer, qw, sw = make_layer(W, bias)
    y, qa, sa = run_fused(layer, A)
    check_rows(y, qa, sa, qw, sw, bias, np.arange(M))


def test_special_rows():
    """All-zero and all -0 rows (S = 1), a constant row, rows whose amax is
    below 2^-64 (exact-division quotient, reciprocal 0), bf16 subnormals, in a
    ragged 300 x 2064 activation spanning two pair tiles."""
    M, N, K = 300, 264, 2064
    A = synth.normal_bf16("gpu/fused/special/A", (M, K), 1.0, outlier_p=0.01, outlier_factor=30.0).copy()
    A[0] = 0x0000                       # +0
    A[1] = 0x8000                       # -0
    A[2] = 0x3F00                       # 0.5 everywhere
    tiny = synth.normal_bf16("gpu/fused/special/tiny", (4, K), 1.0)
    f = synth.bf16_to_f32(tiny) * np.float32(2.0 ** -70)
    A[3:7] = (f.view(np.uint32) >> 16).astype(np.uint16)  # amax ~ 2^-68 (truncated to bf16)
    A[7] = np.where(np.arange(K) % 2 == 0, 0x0001, 0x8003).astype(np.uint16)  # bf16 subnormals only
    A[257] = 0x0000                     # a zero row in the second pair tile
    W = synth.normal_bf16("gpu/fused/special/W", (N, K), 0.02)
    bias = synth.normal_bf16("gpu/fused/special/b", (N,), 0.1)
    layer, qw, sw = make_layer(W, bias)
    y, qa, sa = run_fused(layer, A)
    assert sa[0] == 1.0 and sa[1] == 1.0 and sa[257] == 1.0
    check_rows(y, qa, sa, qw, sw, bias, np.arange(M))


def test_argument_errors_launch_nothing():
    L = fp8.load_library()
    W = synth.normal_bf16("gpu/fused/err/W", (64, 128), 0.02)
    layer, _, _ = make_layer(W, None)
    a = to_device_bf16(synth.normal_bf16("gpu/fused/err/A", (16, 128), 1.0))
    y = torch.empty((16, 64), dtype=torch.bfloat16, device="cuda")
    sc = torch.empty((64,), dtype=torch.float32, device="cuda")
    s = fp8._stream(a.device)
    assert L.fp8_scaled_linear_fused(layer.handle, 16, a.data_ptr(), None, y.data_ptr(), s) == 1
    assert L.fp8_scaled_linear_fused(layer.handle, 16, a.data_ptr(), sc.data_ptr() + 2, y.data_ptr(), s) == 1
    assert L.fp8_scaled_linear_fused(layer.handle, 16, a.data_ptr() + 8, sc.data_ptr(), y.data_ptr(), s) == 1
    assert L.fp8_scaled_linear_fused(layer.handle, -1, a.data_ptr(), sc.data_ptr(), y.data_ptr(), s) == 1
    assert L.fp8_scaled_linear_fused(layer.handle, 0, None, None, None, s) == 0
    assert L.fp8_scaled_linear_fused(None, 16, a.data_ptr(), sc.data_ptr(), y.data_ptr(), s) == 1
    torch.cuda.synchronize()
    assert fp8.device_error() == 0


@pytest.mark.parametrize("M,N,K", [(200, 264, 16384), (37, 24, 8208)])
def test_long_rows_two_pass_scale_prepass(M, N, K):
    """Rows longer than 8192 elements take the two-pass row-scale pre-pass
    (scales only, no codes written)."""
    A = synth.normal_bf16(f"gpu/fused/long/A/{M}x{K}", (M, K), 1.0, outlier_p=0.01, outlier_factor=20.0)
    W = synth.normal_bf16(f"gpu/fused/long/W/{N}x{K}", (N, K), 0.02)
    bias = synth.normal_bf16(f"gpu/fused/long/b/{N}", (N,), 0.1)
    layer, qw, sw = make_layer(W, bias)
    y, qa, sa = run_fused(layer, A)
    check_rows(y, qa, sa, qw, sw, bias, np.arange(M))
