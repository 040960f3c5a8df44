"""Pins for the oracle's per-tensor quantiser on fp16 and fp32 tensors (CPU only).

The state-dict node of "Quantize Model to FP8 Format" takes a model's weights
in whatever floating precision they hold. Checked against: hand-worked
tensors (tests/golden/quant_tensor_f16_f32.txt) whose values are not exact in
bf16, with the scale rounded to fp32 here by exact rational arithmetic; the
binary16 decode against numpy's float16 conversion on all 65536 patterns; the
same recipe spelt with PyTorch CPU ops; and agreement with the bf16 quantiser
when the values are exact in bf16.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synth
from conftest import read_golden
from test_oracle_quant import FMTS, TORCH_DT, fp32_round_exact

SRC_NP = {"f32": np.float32, "f16": np.float16}


@pytest.mark.parametrize("row", read_golden("quant_tensor_f16_f32.txt"), ids=lambda r: r[0])
def test_hand_worked_tensors(row):
    sep = row.index("|")
    fmt, src, scale = FMTS[row[1]], SRC_NP[row[2]], row[3]
    pairs = [p.split(":") for p in row[sep + 1:]]
    vals = [float.fromhex(v) for v, _ in pairs]
    x = np.array(vals, dtype=src)
    assert [float(v) for v in x] == vals, "fixture values must be exact in the source dtype"
    codes = np.array([int(c, 16) for _, c in pairs], dtype=np.uint8)
    q, s = oracle.quantize_tensor_typed(x, fmt)
    assert np.float32(s) == fp32_round_exact(Fraction(scale)), (s, scale)
    assert np.array_equal(q, codes), (q, codes)


def test_f16_decode_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float32)
    got = np.array([oracle.f16_to_f32(int(b)) for b in bits], dtype=np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))  # signed zeros included


def torch_quantize_tensor(x: torch.Tensor, fmt: int):
    x = x.float()
    amax = x.abs().amax()
    s = torch.ones(()) if amax == 0 else amax / torch.tensor(oracle.FMAX[fmt], dtype=torch.float32)
    return (x / s).to(TORCH_DT[fmt]).view(torch.uint8).numpy(), float(s)


@pytest.mark.parametrize("fmt", [oracle.E4M3FN, oracle.E5M2])
@pytest.mark.parametrize("src", ["f32", "f16"])
def test_matches_torch_recipe(fmt, src):
    rng = np.random.default_rng(7)
    x = (rng.standard_normal(20000) * 0.02).astype(SRC_NP[src])
    x[rng.integers(0, x.size, 20)] *= 50
    x[:3] = [0.0, -0.0, 2.0 ** -20]
    q, s = oracle.quantize_tensor_typed(x, fmt)
    qt, st = torch_quantize_tensor(torch.from_numpy(x), fmt)
    assert np.float32(s) == np.float32(st)
    assert np.array_equal(q, qt)


@pytest.mark.parametrize("fmt", [oracle.E4M3FN, oracle.E5M2])
def test_bf16_exact_values_agree_across_dtypes(fmt):
    """Values exact in bf16 (and in fp16's range): the same codes and scale from
    every source dtype."""
    a = synth.state_dict_tensor("test/tensor_dtypes", (64, 96))
    f32 = synth.bf16_to_f32(a)
    q0, s0 = oracle.quantize_tensor(a, fmt)
    q1, s1 = oracle.quantize_tensor_typed(a, fmt)
    q2, s2 = oracle.quantize_tensor_typed(f32, fmt)
    f16 = f32.astype(np.float16)
    exact16 = f16.astype(np.float32) == f32
    assert exact16.mean() > 0.99  # N(0, 0.02) weights: nearly all exact in fp16 too
    q3, s3 = oracle.quantize_tensor_typed(np.where(exact16, f16, np.float16(0)), fmt)
    q4, s4 = oracle.quantize_tensor_typed(np.where(exact16, f32, np.float32(0)), fmt)
    assert s0 == s1 == s2 and np.array_equal(q0, q1) and np.array_equal(q0, q2)
    assert s3 == s4 and np.array_equal(q3, q4)


def test_zero_tensor_gets_unit_scale():
    for dt in (np.float16, np.float32):
        q, s = oracle.quantize_tensor_typed(np.zeros((3, 5), dtype=dt), oracle.E4M3FN)
        assert s == 1.0 and np.all(q == 0)
