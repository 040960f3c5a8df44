"""Producer fusion on the GPU: bf16(act(h)) quantised per token in one kernel.

The activation is evaluated in fp32 with CUDA's erfcf / expf, so its bf16
result may differ from the oracle's correctly rounded double activation by one
bf16 ulp where the true value sits next to a rounding boundary; every element
must be within one ulp and such differences must be rare. The codes and scales
must then equal, bit for bit, the oracle's quantisation of the GPU's own bf16
activation."""
import numpy as np
import pytest
import torch

import oracle
import synth
from conftest import to_device_bf16, to_host_u16

pytestmark = pytest.mark.gpu

fp8 = pytest.importorskip("dit_rowwise_amax_b200")

KINDS = {"gelu": oracle.ACT_GELU_ERF, "gelu_tanh": oracle.ACT_GELU_TANH, "silu": oracle.ACT_SILU}


def ordered(b: np.ndarray) -> np.ndarray:
    b = b.astype(np.int64)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def check(h: np.ndarray, act: str):
    q, s, g = fp8.act_quantize_rowwise(to_device_bf16(h), act, return_bf16=True)
    q2, s2 = fp8.act_quantize_rowwise(to_device_bf16(h), act)
    torch.cuda.synchronize()
    g_gpu = to_host_u16(g)
    g_ref = oracle.act_bf16(KINDS[act], h)
    ulps = np.abs(ordered(g_gpu) - ordered(g_ref))
    assert ulps.max() <= 1, f"{act}: activation off by {ulps.max()} bf16 ulps"
    assert np.mean(ulps != 0) < 2e-3, f"{act}: {np.mean(ulps != 0):.2e} of elements differ by one ulp"
    qo, so = oracle.quantize_rows(g_gpu, oracle.E4M3FN)
    assert np.array_equal(s.cpu().numpy(), so)
    assert np.array_equal(q.cpu().numpy(), qo)
    assert torch.equal(q, q2) and torch.equal(s, s2), "output differs when the bf16 activation is not stored"


@pytest.mark.parametrize("act", list(KINDS))
def test_ffn_down_input_full_size(act):
    """[4096, 8192]: the FFN-up output shape that feeds FFN-down."""
    h = synth.normal_bf16("gpu/act/h", (4096, 8192), 1.0, outlier_p=1e-3, outlier_factor=8.0)
    check(h, act)


@pytest.mark.parametrize("M,K", [(1, 16), (129, 2064), (37, 16384), (300, 272)])
def test_ragged_and_two_pass(M, K):
    h = synth.normal_bf16(f"gpu/act/r/{M}x{K}", (M, K), 3.0)
    for act in KINDS:
        check(h, act)


def test_fused_chain_matches_separate_steps():
    """GELU-quantise then the FFN-down GEMM from the (codes, scale) pair equals
    quantising the stored bf16 GELU output and multiplying it."""
    d = synth.ffn_down()
    layer = fp8.FP8Linear.from_weight(to_device_bf16(d["W"][:512]), to_device_bf16(d["bias"][:512]))
    h = to_device_bf16(synth.normal_bf16("gpu/act/chain", (256, 8192), 1.0))
    q, s, g = fp8.act_quantize_rowwise(h, "gelu", return_bf16=True)
    y_fused = layer.forward_fp8(q, s)
    y_sep = layer.forward(g)
    torch.cuda.synchronize()
    assert torch.equal(y_fused.view(torch.int16), y_sep.view(torch.int16))
