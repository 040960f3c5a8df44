"""FP8 weight-only linear on the GPU (bf16 activation, E4M3 weight decoded to
bf16 in shared memory, BF16 tensor cores) vs the CPU oracle's double-precision
product of the same bf16 activation and decoded weight:
|gpu - ref| <= 1e-2 |ref| + 1e-3 rms(ref)."""
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


def check_rows(y, A, qw, sw, bias, rows):
    ref = oracle.linear_weight_only(np.ascontiguousarray(A[rows]), qw, sw, bias)
    got = bf16_tensor_to_f64(y)[rows]
    ok, worst = oracle.tolerance_ok(got, ref)
    assert ok, f"tolerance exceeded: worst error / bound = {worst:.3f}"


@pytest.mark.parametrize("cfg", ["ffn_up", "ffn_down"])
def test_ffn_full_size(cfg):
    """Every output of both FFN layers (4096 rows, the 256 x 256 pair plan)."""
    d = getattr(synth, cfg)()
    layer, qw, sw = make_layer(d["W"], d["bias"])
    y = layer.forward_weight_only(to_device_bf16(d["A"]))
    torch.cuda.synchronize()
    check_rows(y, d["A"], qw, sw, d["bias"], np.arange(d["A"].shape[0]))


def test_tiny_config_full():
    d = synth.tiny()
    layer, qw, sw = make_layer(d["W"], d["bias"])
    y = layer.forward_weight_only(to_device_bf16(d["A"]))
    torch.cuda.synchronize()
    check_rows(y, d["A"], qw, sw, d["bias"], np.arange(64))


@pytest.mark.parametrize("M", [1, 26, 129, 257, 300])
@pytest.mark.parametrize("N,K", [(8, 16), (136, 48), (520, 2064), (2048, 2048)])
def test_ragged_shapes(M, N, K):
    A = synth.normal_bf16(f"gpu/wo/A/{M}x{K}", (M, K), 1.0, outlier_p=0.01, outlier_factor=20.0)
    W = synth.normal_bf16(f"gpu/wo/W/{N}x{K}", (N, K), 0.02)
    bias = synth.normal_bf16(f"gpu/wo/b/{N}", (N,), 0.1)
    layer, qw, sw = make_layer(W, bias)
    y = layer.forward_weight_only(to_device_bf16(A))
    torch.cuda.synchronize()
    check_rows(y, A, qw, sw, bias, np.arange(M))


def test_closed_form_constant_operands():
    """A = 1.0 everywhere, W row n constant: y[m, n] = K dec(code_n) sw[n]."""
    M, N, K = 300, 256, 1024
    A = np.full((M, K), 0x3F80, dtype=np.uint16)
    vals = np.linspace(-2.0, 2.0, N).astype(np.float32)
    W = np.repeat(((vals.view(np.uint32) + 0x8000) >> 16).astype(np.uint16)[:, None], K, axis=1)
    layer, qw, sw = make_layer(W, None)
    y = layer.forward_weight_only(to_device_bf16(A))
    torch.cuda.synchronize()
    dec = oracle.decode_table(oracle.E4M3FN)[qw[:, 0]]
    expect = np.broadcast_to(K * dec * sw.astype(np.float64), (M, N))
    ok, worst = oracle.tolerance_ok(bf16_tensor_to_f64(y), expect)
    assert ok, worst
