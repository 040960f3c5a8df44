"""Pins for the oracle's FP8 codec (CPU only).

The oracle's decode/encode are checked against things other than
themselves: hand-typed anchor codes and hand-worked rounding cases
(tests/golden), PyTorch's own float8_e4m3fn / float8_e5m2 dtypes (an
independent library), and a brute-force nearest-code search.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from conftest import read_golden

FMTS = {"e4m3fn": oracle.E4M3FN, "e5m2": oracle.E5M2}
TORCH_DT = {oracle.E4M3FN: torch.float8_e4m3fn, oracle.E5M2: torch.float8_e5m2}
MAX_CODE = {oracle.E4M3FN: 0x7E, oracle.E5M2: 0x7B}


def _parse_value(s: str) -> float:
    if s == "-0":
        return -0.0
    return float(s)


def torch_decode_table(fmt: int) -> np.ndarray:
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(TORCH_DT[fmt]).to(torch.float64).numpy()


@pytest.mark.parametrize("row", read_golden("fp8_anchor_codes.txt"), ids=lambda r: f"{r[0]}-{r[1]}")
def test_anchor_codes(row):
    fmt, code, value = FMTS[row[0]], int(row[1], 16), _parse_value(row[2])
    got = oracle.decode(fmt, code)
    if math.isnan(value):
        assert math.isnan(got)
    else:
        assert got == value
        assert math.copysign(1.0, got) == math.copysign(1.0, value)


@pytest.mark.parametrize("fmt", [oracle.E4M3FN, oracle.E5M2])
def test_decode_matches_torch_dtype(fmt):
    ours = oracle.decode_table(fmt)
    ref = torch_decode_table(fmt)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))


@pytest.mark.parametrize("fmt", [oracle.E4M3FN, oracle.E5M2])
def test_decode_monotone_and_symmetric(fmt):
    t = oracle.decode_table(fmt)
    pos = t[: MAX_CODE[fmt] + 1]
    assert np.all(np.diff(pos) > 0)
    assert pos[-1] == oracle.FMAX[fmt]
    for c in range(MAX_CODE[fmt] + 1):
        assert t[c | 0x80] == -t[c]


@pytest.mark.parametrize("row", read_golden("encode_cases.txt"), ids=lambda r: f"{r[0]}:{r[1]}")
def test_hand_worked_encodes(row):
    fmt, v, code = FMTS[row[0]], np.float32(_parse_value(row[1])), int(row[2], 16)
    assert int(oracle.encode(fmt, np.array([v]))[0]) == code


def brute_force_encode(fmt: int, v: np.ndarray) -> np.ndarray:
    """Nearest finite code by exhaustive search over all codes of v's sign;
    exact ties go to the even code; |v| above fmax saturates."""
    table = torch_decode_table(fmt)
    maxc = MAX_CODE[fmt]
    pos_vals = table[: maxc + 1]
    out = np.empty(v.shape, dtype=np.uint8)
    a = np.abs(v.astype(np.float64))
    sign = np.where(np.signbit(v), 0x80, 0).astype(np.uint8)
    for lo in range(0, v.size, 4096):
        aa = a[lo: lo + 4096]
        d = np.abs(aa[:, None] - pos_vals[None, :])
        dmin = d.min(axis=1, keepdims=True)
        is_min = d == dmin
        idx = np.arange(maxc + 1)[None, :]
        # among minima prefer the even code (lowest mantissa bit 0)
        score = np.where(is_min, np.where(idx % 2 == 0, 0, 1), 2)
        best = np.argmin(score, axis=1).astype(np.uint8)
        best = np.where(aa > pos_vals[-1], maxc, best)
        out[lo: lo + 4096] = best
    return out | sign


def interesting_fp32(fmt: int, n_random: int = 200_000, seed: int = 1) -> np.ndarray:
    """All finite bf16 patterns, random log-uniform fp32 values, and every
    midpoint between adjacent codes with its fp32 neighbours."""
    bf = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)
    bf = bf[np.isfinite(bf)]
    rng = np.random.default_rng(seed)
    fmax = oracle.FMAX[fmt]
    mag = np.exp2(rng.uniform(math.log2(fmax) - 30, math.log2(fmax) + 2, n_random))
    rnd = (mag * rng.choice([-1.0, 1.0], n_random)).astype(np.float32)
    t = torch_decode_table(fmt)[: MAX_CODE[fmt] + 1]
    mids = ((t[1:] + t[:-1]) / 2).astype(np.float32)
    mids = np.concatenate([mids, [np.float32(fmax + (fmax - t[-2]) / 2)]])
    near = np.concatenate([mids, np.nextafter(mids, np.float32(np.inf)), np.nextafter(mids, np.float32(0))])
    near = np.concatenate([near, -near])
    return np.concatenate([bf, rnd, near]).astype(np.float32)


@pytest.mark.parametrize("fmt", [oracle.E4M3FN, oracle.E5M2])
def test_encode_equals_brute_force(fmt):
    v = interesting_fp32(fmt)
    got = oracle.encode(fmt, v)
    ref = brute_force_encode(fmt, v)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(v[i]), hex(got[i]), hex(ref[i])) for i in bad[:10]]


@pytest.mark.parametrize("fmt", [oracle.E4M3FN, oracle.E5M2])
def test_encode_matches_torch_cast_in_range(fmt):
    """PyTorch's fp32 -> float8 cast rounds to nearest-even; it does not
    saturate, so only |v| <= fmax is compared."""
    v = interesting_fp32(fmt, seed=2)
    v = v[np.abs(v.astype(np.float64)) <= oracle.FMAX[fmt]]
    ref = torch.from_numpy(v).to(TORCH_DT[fmt]).view(torch.uint8).numpy()
    got = oracle.encode(fmt, v)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(v[i]), hex(got[i]), hex(ref[i])) for i in bad[:10]]


@pytest.mark.parametrize("fmt", [oracle.E4M3FN, oracle.E5M2])
def test_encode_round_trips_every_finite_code(fmt):
    t = oracle.decode_table(fmt)
    codes = np.array([c for c in range(256) if np.isfinite(t[c])], dtype=np.uint8)
    got = oracle.encode(fmt, t[codes].astype(np.float32))
    assert np.array_equal(got, codes)


def test_encode_special_values():
    v = np.array([np.inf, -np.inf, np.nan], dtype=np.float32)
    assert list(oracle.encode(oracle.E4M3FN, v)) == [0x7E, 0xFE, 0x7F]
    assert list(oracle.encode(oracle.E5M2, v)) == [0x7B, 0xFB, 0x7F]
