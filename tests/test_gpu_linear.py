"""FP8 linear (quantise -> tcgen05 GEMM -> scale / bias / bf16) on the GPU vs
the CPU oracle.

The oracle multiplies its own FP8 codes after the test has asserted they
equal the GPU's, then the bf16 outputs must satisfy
|gpu - ref| <= 1e-2 |ref| + 1e-3 rms(ref) elementwise."""
import numpy as np
import pytest
import torch

import oracle
import synth
from conftest import bf16_tensor_to_f64, canary_buffer, check_canary, to_device_bf16

pytestmark = pytest.mark.gpu

fp8 = pytest.importorskip("dit_rowwise_amax_b200")


def make_layer(W, bias):
    """GPU per-channel weight prep, checked bit-exact against the oracle."""
    qw, sw = fp8.quantize_weight_per_channel(to_device_bf16(W))
    b = None if bias is None else to_device_bf16(bias)
    layer = fp8.FP8Linear(qw, sw, b)
    torch.cuda.synchronize()
    qo, so = oracle.quantize_rows(W, oracle.E4M3FN)
    assert np.array_equal(qw.cpu().numpy(), qo) and np.array_equal(sw.cpu().numpy(), so)
    return layer, qo, so


def run_bf16(layer, A):
    M, K = A.shape
    qa = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    sa = torch.empty((M,), dtype=torch.float32, device="cuda")
    y = layer.forward(to_device_bf16(A), qa_scratch=qa, sa_scratch=sa)
    torch.cuda.synchronize()
    qao, sao = oracle.quantize_rows(A, oracle.E4M3FN)
    assert np.array_equal(qa.cpu().numpy(), qao), "activation codes differ"
    assert np.array_equal(sa.cpu().numpy(), sao), "activation scales differ"
    return y, qao, sao


def check_full(y, qa, sa, qw, sw, bias):
    ref = oracle.linear(qa, sa, qw, sw, bias)
    got = bf16_tensor_to_f64(y)
    ok, worst = oracle.tolerance_ok(got, ref)
    assert ok, f"tolerance exceeded: worst error / bound = {worst:.3f}"
    return worst


def test_tiny_config_full():
    d = synth.tiny()
    layer, qw, sw = make_layer(d["W"], d["bias"])
    y, qa, sa = run_bf16(layer, d["A"])
    check_full(y, qa, sa, qw, sw, d["bias"])
    y_call = layer(to_device_bf16(d["A"]))  # the layer is callable like a torch module
    torch.cuda.synchronize()
    assert torch.equal(y_call.view(torch.int16), y.view(torch.int16))


def test_ffn_up_full_size():
    """Every one of the 4096 x 8192 outputs against the oracle's exact product."""
    d = synth.ffn_up()
    layer, qw, sw = make_layer(d["W"], d["bias"])
    y, qa, sa = run_bf16(layer, d["A"])
    check_full(y, qa, sa, qw, sw, d["bias"])


def test_ffn_down_full_size():
    """Every one of the 4096 x 2048 outputs (K = 8192) against the oracle."""
    d = synth.ffn_down()
    layer, qw, sw = make_layer(d["W"], d["bias"])
    y, qa, sa = run_bf16(layer, d["A"])
    check_full(y, qa, sa, qw, sw, d["bias"])


@pytest.mark.parametrize("M", [1, 26, 127, 128, 129, 255, 700])
@pytest.mark.parametrize("N,K", [(512, 256), (520, 2064), (2048, 2048), (136, 48), (256, 16)])
def test_ragged_shapes(M, N, K):
    A = synth.normal_bf16(f"gpu/lin/A/{M}x{K}", (M, K), 1.0, outlier_p=0.01, outlier_factor=20.0)
    W = synth.normal_bf16(f"gpu/lin/W/{N}x{K}", (N, K), 0.02)
    bias = synth.normal_bf16(f"gpu/lin/b/{N}", (N,), 0.1)
    layer, qw, sw = make_layer(W, bias)
    y, qa, sa = run_bf16(layer, A)
    check_full(y, qa, sa, qw, sw, bias)


@pytest.mark.parametrize("M,N,K", [(300, 8, 16), (200, 24, 16384), (513, 264, 4112), (257, 2048, 2048)])
def test_extreme_shapes(M, N, K):
    """Smallest N, the longest K (two-pass quantiser, 128 k-blocks), K not a
    multiple of the 128-wide k-block, and M just past a 256-row pair tile."""
    A = synth.normal_bf16(f"gpu/ext/A/{M}x{K}", (M, K), 1.0, outlier_p=0.01, outlier_factor=20.0)
    W = synth.normal_bf16(f"gpu/ext/W/{N}x{K}", (N, K), 0.02)
    bias = synth.normal_bf16(f"gpu/ext/b/{N}", (N,), 0.1)
    layer, qw, sw = make_layer(W, bias)
    y, qa, sa = run_bf16(layer, A)
    check_full(y, qa, sa, qw, sw, bias)


def test_no_bias():
    d = synth.tiny()
    layer, qw, sw = make_layer(d["W"], None)
    y, qa, sa = run_bf16(layer, d["A"])
    check_full(y, qa, sa, qw, sw, None)


def test_prequantised_input_equals_bf16_path():
    d = synth.ffn_up()
    layer, qw, sw = make_layer(d["W"], d["bias"])
    A = d["A"][:1000]
    y1, qa, sa = run_bf16(layer, A)
    y2 = layer.forward_fp8(torch.from_numpy(qa).cuda(), torch.from_numpy(sa).cuda())
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_multi_equals_single_calls_attention_full_size():
    d = synth.attention()
    layers, refs = [], []
    for p in ("q", "k", "v"):
        layer, qw, sw = make_layer(d[f"W_{p}"], d[f"bias_{p}"])
        layers.append(layer)
        refs.append((qw, sw, d[f"bias_{p}"]))
    for name in ("hidden", "encoder"):
        A = d[name]
        x = to_device_bf16(A)
        M = A.shape[0]
        qa = torch.empty((M, 2048), dtype=torch.uint8, device="cuda")
        sa = torch.empty((M,), dtype=torch.float32, device="cuda")
        ys = fp8.scaled_linear_multi(layers, x, qa_scratch=qa, sa_scratch=sa)
        singles = [l.forward(x) for l in layers]
        torch.cuda.synchronize()
        qao, sao = oracle.quantize_rows(A, oracle.E4M3FN)
        assert np.array_equal(qa.cpu().numpy(), qao) and np.array_equal(sa.cpu().numpy(), sao)
        for y, ys_ref, (qw, sw, b) in zip(ys, singles, refs):
            assert torch.equal(y.view(torch.int16), ys_ref.view(torch.int16))
            check_full(y, qao, sao, qw, sw, b)  # all 32760 x 2048 outputs of each projection


@pytest.mark.parametrize("M", [26, 333])  # one row tile (A loaded as 32 rows) / three row tiles
def test_multi_two_and_four_layers_with_different_n(M):
    K = 512
    A = synth.normal_bf16("gpu/multi/A" if M == 333 else f"gpu/multi/A{M}", (M, K), 1.0)
    layers, refs = [], []
    for i, N in enumerate((256, 520, 136, 1024)):
        W = synth.normal_bf16(f"gpu/multi/W{i}", (N, K), 0.02)
        b = synth.normal_bf16(f"gpu/multi/b{i}", (N,), 0.1)
        layer, qw, sw = make_layer(W, b)
        layers.append(layer)
        refs.append((qw, sw, b))
    x = to_device_bf16(A)
    qao, sao = oracle.quantize_rows(A, oracle.E4M3FN)
    for n in (2, 4):
        assert layers[0].plan(M, n)[:2] == (128, 64)  # the tiles of all n layers fit one wave
        ys = fp8.scaled_linear_multi(layers[:n], x)
        torch.cuda.synchronize()
        for y, (qw, sw, b) in zip(ys, refs[:n]):
            check_full(y, qao, sao, qw, sw, b)
        singles = [layer.forward(x) for layer in layers[:n]]
        torch.cuda.synchronize()
        for y, s1 in zip(ys, singles):
            assert torch.equal(y.view(torch.int16), s1.view(torch.int16))


def test_output_canaries():
    M, N, K = 129, 520, 272
    A = synth.normal_bf16("gpu/canary/A", (M, K), 1.0)
    W = synth.normal_bf16("gpu/canary/W", (N, K), 0.02)
    layer, qw, sw = make_layer(W, None)
    ybuf, yb = canary_buffer(M * N * 2)
    y = yb.view(torch.bfloat16).view(M, N)
    layer.forward(to_device_bf16(A), y=y)
    torch.cuda.synchronize()
    check_canary(ybuf, M * N * 2)
    qa, sa = oracle.quantize_rows(A, oracle.E4M3FN)
    check_full(y, qa, sa, qw, sw, None)


def test_closed_form_constant_rows():
    """A = all ones -> codes 0x7E, S = fp32(1/448); W row n constant c_n ->
    y[m, n] = K * dec(c_n) * sw[n] * (448 * S) + bias[n]."""
    M, N, K = 64, 256, 1024
    A = np.full((M, K), 0x3F80, dtype=np.uint16)
    vals = np.linspace(-2.0, 2.0, N).astype(np.float32)
    W = np.repeat(((vals.view(np.uint32) + 0x8000) >> 16).astype(np.uint16)[:, None], K, axis=1)
    layer, qw, sw = make_layer(W, None)
    y, qa, sa = run_bf16(layer, A)
    assert np.all(qa == 0x7E)
    dec = oracle.decode_table(oracle.E4M3FN)[qw[:, 0]]
    expect = K * dec[None, :] * sw[None, :].astype(np.float64) * (448.0 * np.float64(sa[0]))
    ok, worst = oracle.tolerance_ok(bf16_tensor_to_f64(y), np.broadcast_to(expect, (M, N)))
    assert ok, worst


def test_plan_is_reported():
    d = synth.ffn_up()
    layer, _, _ = make_layer(d["W"][:256], d["bias"][:256])
    bm, bn, ctas = layer.plan(4096)
    assert bm == 128 and bn in (64, 128, 256) and ctas >= 1
