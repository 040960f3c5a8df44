"""Pins for the oracle's amax quantisers (CPU only).

Checked against: hand-worked rows (tests/golden/quant_rows.txt) with the
scale rounded to fp32 here by exact rational arithmetic; the same recipe
spelled with PyTorch CPU ops (torch's fp32 division and its float8 cast, an
independent library); and invariants of the method (the amax element maps
to +-fmax, an all-zero row gets S = 1, round-trip error within half a code
step, per-tensor equals rowwise over the flattened tensor).
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synth
from conftest import read_golden

FMTS = {"e4m3fn": oracle.E4M3FN, "e5m2": oracle.E5M2}
TORCH_DT = {oracle.E4M3FN: torch.float8_e4m3fn, oracle.E5M2: torch.float8_e5m2}


def fp32_round_exact(fr: Fraction) -> np.float32:
    """Round a positive rational to the nearest fp32 (ties to even), exactly."""
    assert fr > 0
    e = fr.numerator.bit_length() - fr.denominator.bit_length()
    while Fraction(2) ** e > fr:
        e -= 1
    while Fraction(2) ** (e + 1) <= fr:
        e += 1
    e = max(e, -126)  # subnormal range keeps the smallest binade's spacing
    step = Fraction(2) ** (e - 23)
    q, r = divmod(fr, step)
    q = int(q)
    if r > step / 2 or (r == step / 2 and q % 2 == 1):
        q += 1
    return np.float32(float(q * step))


def to_bf16_exact(values) -> np.ndarray:
    f = np.asarray(values, dtype=np.float32)
    bits = f.view(np.uint32)
    assert np.all(bits & 0xFFFF == 0), "fixture values must be exact in bf16"
    return (bits >> 16).astype(np.uint16)


@pytest.mark.parametrize("row", read_golden("quant_rows.txt"), ids=lambda r: r[0])
def test_hand_worked_rows(row):
    sep = row.index("|")
    fmt = FMTS[row[1]]
    scale = row[2]
    pairs = [p.split(":") for p in row[sep + 1:]]
    x = to_bf16_exact([float(v) for v, _ in pairs])[None, :]
    codes = np.array([int(c, 16) for _, c in pairs], dtype=np.uint8)
    q, s = oracle.quantize_rows(x, fmt)
    expect_s = np.float32(1.0) if scale == "1" else fp32_round_exact(Fraction(scale))
    assert s[0] == expect_s, (s[0], expect_s)
    assert np.array_equal(q[0], codes), (q[0], codes)


def torch_quantize_rows(x_bf16: np.ndarray, fmt: int):
    x = torch.from_numpy(x_bf16.astype(np.int16)).view(torch.bfloat16).float()
    amax = x.abs().amax(dim=1)
    s = amax / torch.tensor(oracle.FMAX[fmt], dtype=torch.float32)
    s = torch.where(amax == 0, torch.ones_like(s), s)
    q = (x / s[:, None]).to(TORCH_DT[fmt]).view(torch.uint8)
    return q.numpy(), s.numpy()


@pytest.mark.parametrize("fmt", [oracle.E4M3FN, oracle.E5M2])
def test_rows_match_torch_recipe(fmt):
    x = synth.tiny()["A"]
    extra = synth.normal_bf16("test/quant_rows", (300, 272), 3.0, outlier_p=0.01, outlier_factor=40.0)
    for a in (x, extra):
        q, s = oracle.quantize_rows(a, fmt)
        qt, st = torch_quantize_rows(a, fmt)
        assert np.array_equal(s, st)
        assert np.array_equal(q, qt)


@pytest.mark.parametrize("fmt", [oracle.E4M3FN, oracle.E5M2])
def test_rows_invariants(fmt):
    a = synth.normal_bf16("test/quant_inv", (128, 512), 0.7, outlier_p=0.02, outlier_factor=25.0)
    a[5] = 0  # all-zero row
    a[6] = to_bf16_exact([-1.75] * 512)  # constant row
    q, s = oracle.quantize_rows(a, fmt)
    x = synth.bf16_to_f32(a).astype(np.float64)
    table = oracle.decode_table(fmt)
    fmax = oracle.FMAX[fmt]
    maxcode = 0x7E if fmt == oracle.E4M3FN else 0x7B
    assert s[5] == 1.0 and np.all(q[5] == 0)
    assert np.all(q[6] == (maxcode | 0x80))
    for m in range(a.shape[0]):
        if m == 5:
            continue
        i = int(np.argmax(np.abs(x[m])))
        assert q[m, i] & 0x7F == maxcode
        # round-trip: |dec(q) - x/S| <= half the local code step (+ fp32 quotient rounding)
        quot = x[m] / float(s[m])
        dec = table[q[m]]
        mb = 3 if fmt == oracle.E4M3FN else 2
        emin = -6 if fmt == oracle.E4M3FN else -14
        e = np.maximum(np.floor(np.log2(np.maximum(np.abs(quot), 1e-300))), emin)
        half_step = np.exp2(e - mb) / 2
        assert np.all(np.abs(dec - quot) <= half_step * (1 + 1e-6) + np.abs(quot) * 2.0 ** -23)
        assert np.all(np.abs(dec) <= fmax)


@pytest.mark.parametrize("fmt", [oracle.E4M3FN, oracle.E5M2])
def test_tensor_equals_single_row(fmt):
    a = synth.state_dict_tensor("test/tensor", (64, 96))
    q, s = oracle.quantize_tensor(a, fmt)
    qr, sr = oracle.quantize_rows(a.reshape(1, -1), fmt)
    assert s == sr[0]
    assert np.array_equal(q.reshape(1, -1), qr)


def test_tensor_zero_gets_unit_scale():
    q, s = oracle.quantize_tensor(np.zeros((4, 8), dtype=np.uint16), oracle.E5M2)
    assert s == 1.0 and np.all(q == 0)
