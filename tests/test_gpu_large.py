"""Sizes beyond 32-bit element indexing: an activation of 2^21 + 5 rows x 1040
(2.18e9 elements, 4.4 GB of bf16), quantised per token and multiplied with a
ragged N = 24 weight (8193 pair tiles in one persistent launch). The inputs
are seeded on the device (torch's generator) so the test needs no 4 GB host
synthesis; sampled rows (the first, the last and random ones) are copied back
and compared with the oracle: codes and scales bit for bit, outputs within
the tolerance."""
import numpy as np
import pytest
import torch

import oracle
import synth
from conftest import bf16_tensor_to_f64, to_device_bf16

pytestmark = pytest.mark.gpu

fp8 = pytest.importorskip("dit_rowwise_amax_b200")

M, K, N = (1 << 21) + 5, 1040, 24


@pytest.fixture(scope="module")
def big():
    if torch.cuda.get_device_properties(0).total_memory < 32 << 30:
        pytest.skip("needs a large-memory GPU")
    g = torch.Generator(device="cuda").manual_seed(1234)
    a = torch.randn((M, K), generator=g, device="cuda").to(torch.bfloat16)
    rng = np.random.default_rng(7)
    rows = np.unique(np.concatenate([np.arange(4), np.arange(M - 4, M), rng.integers(0, M, 56)]))
    host_rows = a[torch.from_numpy(rows).cuda()].cpu().view(torch.int16).numpy().view(np.uint16)
    yield a, rows, host_rows
    del a
    torch.cuda.empty_cache()


def test_quantise_beyond_2g_elements(big):
    a, rows, host_rows = big
    assert a.numel() > (1 << 31)
    q, s = fp8.quantize_rowwise(a)
    torch.cuda.synchronize()
    idx = torch.from_numpy(rows).cuda()
    qo, so = oracle.quantize_rows(host_rows, oracle.E4M3FN)
    assert np.array_equal(q[idx].cpu().numpy(), qo)
    assert np.array_equal(s[idx].cpu().numpy(), so)


def test_linear_8193_pair_tiles(big):
    a, rows, host_rows = big
    W = synth.normal_bf16("gpu/large/W", (N, K), 0.02)
    bias = synth.normal_bf16("gpu/large/b", (N,), 0.1)
    qw, sw = fp8.quantize_weight_per_channel(to_device_bf16(W))
    layer = fp8.FP8Linear(qw, sw, to_device_bf16(bias))
    assert layer.plan(M)[:2] == (256, 256)
    y = layer.forward(a)
    torch.cuda.synchronize()
    assert fp8.device_error() == 0
    qa, sa = oracle.quantize_rows(host_rows, oracle.E4M3FN)
    ref = oracle.linear(qa, sa, qw.cpu().numpy(), sw.cpu().numpy(), bias)
    got = bf16_tensor_to_f64(y[torch.from_numpy(rows).cuda()])
    ok, worst = oracle.tolerance_ok(got, ref)
    assert ok, f"tolerance exceeded: worst error / bound = {worst:.3f}"
