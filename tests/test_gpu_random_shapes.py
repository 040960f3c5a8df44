"""Seeded random shapes through the three linear paths (the FP8 linear from a
bf16 activation, the FP8 weight-only linear, the fused one-launch linear),
each compared elementwise with the oracle on every output. The shapes mix
every tile plan (pair tiles, 128 x 256, 128 x 128, 128 x 64), ragged M, N and
K, and short K (a single k-block) to K = 4096. A second set of few-row shapes
with K up to 9000 runs with a workspace attached, so that the split-K
schedule (FP8 and weight-only) meets ragged shapes too."""
import numpy as np
import pytest
import torch

import oracle
import synth
from conftest import bf16_tensor_to_f64, to_device_bf16

pytestmark = pytest.mark.gpu

fp8 = pytest.importorskip("dit_rowwise_amax_b200")


def shapes(n=40, seed=2024):
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        M = int(rng.integers(1, 1501))
        N = 8 * int(rng.integers(1, 189))
        K = 16 * int(rng.integers(1, 257))
        out.append((M, N, K))
    return out


def check(y, ref):
    ok, worst = oracle.tolerance_ok(bf16_tensor_to_f64(y), ref)
    assert ok, f"tolerance exceeded: worst error / bound = {worst:.3f}"


@pytest.mark.parametrize("M,N,K", shapes())
def test_random_shape_all_paths(M, N, K):
    tag = f"gpu/random/{M}x{N}x{K}"
    A = synth.normal_bf16(tag + "/A", (M, K), 1.0, outlier_p=0.01, outlier_factor=20.0)
    W = synth.normal_bf16(tag + "/W", (N, K), 0.02)
    bias = synth.normal_bf16(tag + "/b", (N,), 0.1)
    qw, sw = fp8.quantize_weight_per_channel(to_device_bf16(W))
    layer = fp8.FP8Linear(qw, sw, to_device_bf16(bias))
    a = to_device_bf16(A)
    y_lin = layer.forward(a)
    y_wo = layer.forward_weight_only(a)
    y_fused = layer.forward_fused(a)
    torch.cuda.synchronize()
    assert fp8.device_error() == 0
    qwn, swn = qw.cpu().numpy(), sw.cpu().numpy()
    qa, sa = oracle.quantize_rows(A, oracle.E4M3FN)
    ref = oracle.linear(qa, sa, qwn, swn, bias)
    check(y_lin, ref)
    check(y_fused, ref)
    check(y_wo, oracle.linear_weight_only(A, qwn, swn, bias))


def small_m_shapes(n=24, seed=2025):
    """Few rows (one or two row tiles) and K up to 9000: the plans where the
    128 x 64 tiles, the short A box and split-K (with a workspace) apply."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        M = int(rng.integers(1, 257))
        N = 8 * int(rng.integers(1, 257))
        K = 16 * int(rng.integers(1, 563))
        out.append((M, N, K))
    return out


@pytest.mark.parametrize("M,N,K", small_m_shapes())
def test_random_small_m_with_workspace(M, N, K):
    tag = f"gpu/random-small/{M}x{N}x{K}"
    A = synth.normal_bf16(tag + "/A", (M, K), 1.0, outlier_p=0.01, outlier_factor=20.0)
    W = synth.normal_bf16(tag + "/W", (N, K), 0.02)
    bias = synth.normal_bf16(tag + "/b", (N,), 0.1)
    qw, sw = fp8.quantize_weight_per_channel(to_device_bf16(W))
    layer = fp8.FP8Linear(qw, sw, to_device_bf16(bias))
    layer.attach_workspace()
    a = to_device_bf16(A)
    y_lin = layer.forward(a)
    y_wo = layer.forward_weight_only(a)
    torch.cuda.synchronize()
    assert fp8.device_error() == 0
    qwn, swn = qw.cpu().numpy(), sw.cpu().numpy()
    qa, sa = oracle.quantize_rows(A, oracle.E4M3FN)
    check(y_lin, oracle.linear(qa, sa, qwn, swn, bias))
    check(y_wo, oracle.linear_weight_only(A, qwn, swn, bias))
