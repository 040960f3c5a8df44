"""Rowwise / per-channel quantiser on the GPU vs the CPU oracle: bit-exact
codes and bit-exact fp32 scales."""
import numpy as np
import pytest
import torch

import oracle
import synth
from conftest import canary_buffer, check_canary, to_device_bf16

pytestmark = pytest.mark.gpu

fp8 = pytest.importorskip("dit_rowwise_amax_b200")


def gpu_quant(a_u16, fmt, ldx=None):
    M, K = a_u16.shape
    if ldx is None or ldx == K:
        x = to_device_bf16(a_u16)
    else:
        padded = np.zeros((M, ldx), dtype=np.uint16)
        padded[:, :K] = a_u16
        x = to_device_bf16(padded)[:, :K]
    q, s = fp8.quantize_rowwise(x, fmt)
    torch.cuda.synchronize()
    return q.cpu().numpy(), s.cpu().numpy()


def assert_same(a_u16, fmt, ldx=None):
    q, s = gpu_quant(a_u16, fmt, ldx)
    qo, so = oracle.quantize_rows(a_u16, fmt)
    assert np.array_equal(s.view(np.uint32), so.view(np.uint32)), "scales differ"
    bad = np.argwhere(q != qo)
    assert bad.size == 0, f"{len(bad)} codes differ, first at {bad[:5].tolist()}"


@pytest.mark.parametrize("fmt", [oracle.E4M3FN, oracle.E5M2])
def test_workload_activations(fmt):
    assert_same(synth.tiny()["A"], fmt)
    assert_same(synth.ffn_up()["A"], fmt)
    assert_same(synth.ffn_down()["A"], fmt)
    att = synth.attention()
    assert_same(att["encoder"], fmt)


def test_attention_hidden_full_size():
    assert_same(synth.attention()["hidden"], oracle.E4M3FN)


@pytest.mark.parametrize("M", [1, 26, 127, 129, 300])
@pytest.mark.parametrize("K", [16, 48, 256, 1040, 2064, 4096, 8192, 8208, 16384])
def test_ragged_shapes(M, K):
    a = synth.normal_bf16(f"gpu/ragged/{M}x{K}", (M, K), 1.5, outlier_p=0.01, outlier_factor=30.0)
    assert_same(a, oracle.E4M3FN)


@pytest.mark.parametrize("ldx", [2048 + 8, 4096])
def test_strided_rows(ldx):
    a = synth.normal_bf16("gpu/strided", (200, 2048), 1.0)
    assert_same(a, oracle.E4M3FN, ldx=ldx)


@pytest.mark.parametrize("fmt", [oracle.E4M3FN, oracle.E5M2])
def test_special_rows(fmt):
    K = 512
    a = synth.normal_bf16("gpu/special", (12, K), 1.0)
    a[0] = 0                                   # all-zero row: S = 1
    a[1] = 0x8000                              # all -0
    a[2] = 0x4040                              # constant 3.0
    a[3] = synth.normal_bf16("gpu/tiny", (K,), 1e-38)   # tiny amax -> subnormal fp32 scale
    a[4, :] = 0x0001                           # smallest bf16 subnormal everywhere
    a[5] = synth.normal_bf16("gpu/huge", (K,), 1e37)    # huge values (finite in bf16)
    a[6, ::2] = 0x7F7F                         # largest finite bf16 mixed in
    a[7] = np.where(np.arange(K) % 3 == 0, 0x3F80, 0xBF80)  # +-1
    assert_same(a, fmt)


def test_all_bf16_patterns_one_row_each_scale():
    """Every finite bf16 value passes through the divide + encode against
    several scales (rows built so the amax is a chosen value)."""
    pats = np.arange(65536, dtype=np.uint32)
    f = (pats << 16).view(np.float32)
    finite = pats[np.isfinite(f)].astype(np.uint16)
    K = 4096
    n = (finite.size + K - 1) // K
    rows = np.zeros((n, K), dtype=np.uint16)
    rows.reshape(-1)[: finite.size] = finite
    for amax_bits in (0x3F80, 0x4120, 0x3C00, 0x7F7F):  # 1, 10, 2^-7, max bf16
        r = rows.copy()
        mag = ((r.astype(np.uint32) << 16).view(np.float32))
        r[np.abs(mag) > ((np.uint32(amax_bits) << 16).view(np.float32))] = 0
        r[:, 0] = amax_bits
        assert_same(r, oracle.E4M3FN)
        assert_same(r, oracle.E5M2)


def test_no_writes_outside_outputs():
    M, K = 129, 2064
    a = synth.normal_bf16("gpu/canary", (M, K), 1.0)
    x = to_device_bf16(a)
    qbuf, q = canary_buffer(M * K)
    sbuf, s_bytes = canary_buffer(M * 4)
    q = q.view(M, K)
    s = s_bytes.view(torch.float32)
    fp8.quantize_rowwise(x, fp8.E4M3FN, q=q, scale=s)
    torch.cuda.synchronize()
    check_canary(qbuf, M * K)
    check_canary(sbuf, M * 4)
    qo, so = oracle.quantize_rows(a, oracle.E4M3FN)
    assert np.array_equal(q.cpu().numpy(), qo)


def test_weight_per_channel_matches_rows():
    for W in (synth.tiny()["W"], synth.ffn_up()["W"], synth.ffn_down()["W"]):
        qw, sw = fp8.quantize_weight_per_channel(to_device_bf16(W))
        torch.cuda.synchronize()
        qo, so = oracle.quantize_rows(W, oracle.E4M3FN)
        assert np.array_equal(sw.cpu().numpy().view(np.uint32), so.view(np.uint32))
        assert np.array_equal(qw.cpu().numpy(), qo)


def test_zero_rows_is_noop():
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    q, s = fp8.quantize_rowwise(x)
    assert q.shape == (0, 64) and s.shape == (0,)


def test_quotient_selftest_exhaustive():
    """Every (bf16 x, bf16 amax) pair, both formats: the quantisers' quotient
    path gives the same FP8 code as IEEE fp32 division (hardware cvt)."""
    assert fp8.selftest_quotient() == (0, 0)
