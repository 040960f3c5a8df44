"""Producer fusion on the GPU: bf16(act(h)) quantised per token in one kernel.

The library evaluates each activation in double and rounds it once to bf16,
so the bf16 activation must equal the oracle's correctly rounded double
activation bit for bit, on every finite bf16 input. The codes and scales must
then equal, bit for bit, the oracle's rowwise quantisation of the oracle's
own activation: quantize_rows(act_bf16(h)), never a quantisation of the GPU's
intermediate."""
import numpy as np
import pytest
import torch

import oracle
import synth
from conftest import to_device_bf16, to_host_u16

pytestmark = pytest.mark.gpu

fp8 = pytest.importorskip("dit_rowwise_amax_b200")

KINDS = {"gelu": oracle.ACT_GELU_ERF, "gelu_tanh": oracle.ACT_GELU_TANH, "silu": oracle.ACT_SILU}


def check(h: np.ndarray, act: str):
    q, s, g = fp8.act_quantize_rowwise(to_device_bf16(h), act, return_bf16=True)
    q2, s2 = fp8.act_quantize_rowwise(to_device_bf16(h), act)
    torch.cuda.synchronize()
    g_ref = oracle.act_bf16(KINDS[act], h)
    g_gpu = to_host_u16(g)
    bad = np.flatnonzero(g_gpu.ravel() != g_ref.ravel())
    assert bad.size == 0, (f"{act}: {bad.size} bf16 activations differ from the oracle, first at input "
                           f"0x{int(h.ravel()[bad[0]]):04x}: gpu 0x{int(g_gpu.ravel()[bad[0]]):04x} "
                           f"oracle 0x{int(g_ref.ravel()[bad[0]]):04x}")
    qo, so = oracle.quantize_rows(g_ref, oracle.E4M3FN)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32)), f"{act}: scales differ"
    assert np.array_equal(q.cpu().numpy(), qo), f"{act}: codes differ"
    assert torch.equal(q, q2) and torch.equal(s, s2), "output differs when the bf16 activation is not stored"


def all_finite_bf16() -> np.ndarray:
    """Every finite bf16 pattern (exponent field != 0xFF), as [255, 256]."""
    b = np.arange(65536, dtype=np.uint32)
    finite = b[((b >> 7) & 0xFF) != 0xFF].astype(np.uint16)
    assert finite.size == 65280
    return finite.reshape(255, 256)


@pytest.mark.parametrize("act", list(KINDS))
def test_activation_table_exhaustive(act):
    """The whole 65536-entry table the kernel reads, through the public entry
    point: every finite bf16 input, stored bf16 activation and codes compared
    with the oracle."""
    check(all_finite_bf16(), act)


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
