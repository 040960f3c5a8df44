"""Pins for the oracle's producer activations and its double -> bf16 rounding
(CPU only): PyTorch's float64 gelu / silu (an independent library), closed
forms, and a brute-force nearest-bf16 search."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth


def bf16_value(bits: int) -> float:
    return float(np.array([bits << 16], dtype=np.uint32).view(np.float32)[0])


@pytest.mark.parametrize("kind,torch_fn", [
    (oracle.ACT_GELU_ERF, lambda t: torch.nn.functional.gelu(t)),
    (oracle.ACT_GELU_TANH, lambda t: torch.nn.functional.gelu(t, approximate="tanh")),
    (oracle.ACT_SILU, lambda t: torch.nn.functional.silu(t)),
])
def test_activation_matches_torch_float64(kind, torch_fn):
    x = np.concatenate([np.linspace(-12, 12, 2001), synth.uniform("act/x", 2000) * 60 - 30, [0.0, -0.0, 1e-30]])
    ref = torch_fn(torch.from_numpy(x)).numpy()
    got = np.array([oracle.act(kind, float(v)) for v in x])
    # torch evaluates 1 + erf / 1 + tanh directly, which cancels for negative x;
    # the oracle's forms do not, hence the small absolute slack.
    assert np.all(np.abs(got - ref) <= 1e-12 * np.abs(ref) + 1e-15)


def test_activation_closed_forms():
    assert oracle.act(oracle.ACT_GELU_ERF, 0.0) == 0.0
    assert oracle.act(oracle.ACT_GELU_ERF, 1.0) == pytest.approx(0.5 * (1 + math.erf(1 / math.sqrt(2))), rel=1e-15)
    assert oracle.act(oracle.ACT_SILU, 2.0) == pytest.approx(2.0 / (1 + math.exp(-2.0)), rel=1e-15)
    assert oracle.act(oracle.ACT_GELU_ERF, 40.0) == 40.0
    assert abs(oracle.act(oracle.ACT_GELU_ERF, -40.0)) < 1e-300


def test_round_bf16_is_nearest_with_ties_to_even():
    rng = np.random.default_rng(3)
    vals = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
                           # exact midpoints between neighbouring bf16 values
                           [bf16_value(b) + (bf16_value(b + 1) - bf16_value(b)) / 2 for b in range(0x3F80, 0x3F90)]])
    for v in vals:
        got = oracle.round_bf16(float(v))
        # brute force over the three bf16 neighbours of the fp32 truncation
        base = int(np.array([abs(v)], dtype=np.float32).view(np.uint32)[0] >> 16)
        cands = [c for c in (base - 1, base, base + 1, base + 2) if 0 <= c < 0x7F80]
        dist = [abs(bf16_value(c) - abs(v)) for c in cands]
        best = min(dist)
        ties = [c for c, d in zip(cands, dist) if d == best]
        expect = min(ties, key=lambda c: (c & 1, c)) | (0x8000 if v < 0 else 0)
        assert got == expect, (v, hex(got), hex(expect))


def test_act_bf16_rounds_the_double_activation():
    h = synth.normal_bf16("act/h", (64, 128), 2.0)
    g = oracle.act_bf16(oracle.ACT_GELU_ERF, h)
    hv = synth.bf16_to_f32(h).astype(np.float64).ravel()
    for i in range(0, hv.size, 97):
        assert g.ravel()[i] == oracle.round_bf16(oracle.act(oracle.ACT_GELU_ERF, hv[i]))
