"""Pins for the oracle's dequantised FP8 GEMM and epilogue (CPU only).

The exact integer dot is checked against Python-integer brute force and
against a float64 numpy matmul of the values decoded by PyTorch's float8
dtype (exact here: every product is a multiple of 2^-18 below 2^18 and
every partial sum stays below 2^35, inside double's 53-bit significand).
The epilogue y = dot * sa * sw + bias is checked on closed forms: constant
operands, an identity-like weight, a sign flip and the bias shift.
"""
import numpy as np
import torch

import oracle
import synth


def torch_decode(codes: np.ndarray) -> np.ndarray:
    return torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def random_codes(shape, seed):
    """Finite E4M3FN codes (NaN codes 0x7F / 0xFF excluded)."""
    rng = np.random.default_rng(seed)
    c = rng.integers(0, 256, size=shape, dtype=np.uint8)
    return np.where((c & 0x7F) == 0x7F, c ^ 0x01, c).astype(np.uint8)


def test_dot_equals_integer_brute_force():
    qa = random_codes((3, 7), 1)
    qw = random_codes((5, 7), 2)
    dot = oracle.dot_units(qa, qw)
    units = lambda c: int(round(float(torch_decode(np.array([c], dtype=np.uint8))[0]) * 512))
    for m in range(3):
        for n in range(5):
            assert dot[m, n] == sum(units(qa[m, k]) * units(qw[n, k]) for k in range(7))


def test_dot_equals_exact_float64_matmul():
    qa = random_codes((40, 2048), 3)
    qw = random_codes((24, 2048), 4)
    ref = torch_decode(qa) @ torch_decode(qw).T  # exact, see module docstring
    assert np.array_equal(oracle.dot_units(qa, qw).astype(np.float64) * 2.0 ** -18, ref)


def test_linear_constant_operands_closed_form():
    K, M, N = 64, 3, 6
    qa = np.full((M, K), 0x38, dtype=np.uint8)  # 1.0
    wcodes = np.array([0x38, 0xB8, 0x40, 0x01, 0x7E, 0x00], dtype=np.uint8)  # 1,-1,2,2^-9,448,0
    qw = np.repeat(wcodes[:, None], K, axis=1)
    sa = np.array([0.5, 0.25, 3.0], dtype=np.float32)
    sw = np.array([2.0, 2.0, 0.5, 1.0, 0.125, 7.0], dtype=np.float32)
    bias_vals = np.array([0.0, 1.0, -2.0, 0.5, 0.0, 3.0], dtype=np.float32)
    bias = (bias_vals.view(np.uint32) >> 16).astype(np.uint16)
    y = oracle.linear(qa, sa, qw, sw, bias)
    wv = np.array([1.0, -1.0, 2.0, 2.0 ** -9, 448.0, 0.0])
    expect = K * wv[None, :] * sa[:, None].astype(np.float64) * sw[None, :] + bias_vals[None, :]
    assert np.array_equal(y, expect)


def test_linear_identity_weight():
    M, K = 5, 32
    qa = random_codes((M, K), 5)
    qw = np.zeros((K, K), dtype=np.uint8)
    qw[np.arange(K), np.arange(K)] = 0x38  # 1.0 on the diagonal
    sa = np.linspace(0.5, 2.0, M).astype(np.float32)
    sw = np.linspace(1.0, 3.0, K).astype(np.float32)
    y = oracle.linear(qa, sa, qw, sw, None)
    expect = torch_decode(qa) * sa[:, None].astype(np.float64) * sw[None, :].astype(np.float64)
    assert np.array_equal(y, expect)


def test_linear_sign_flip_and_bias_shift():
    qa = random_codes((8, 96), 6)
    qw = random_codes((16, 96), 7)
    sa = np.linspace(0.1, 1.0, 8).astype(np.float32)
    sw = np.linspace(0.01, 0.2, 16).astype(np.float32)
    bias = synth.normal_bf16("test/gemm_bias", (16,), 0.1)
    y0 = oracle.linear(qa, sa, qw, sw, None)
    y_neg = oracle.linear(qa, sa, qw ^ 0x80, sw, None)
    assert np.array_equal(y_neg, -y0)
    y_b = oracle.linear(qa, sa, qw, sw, bias)
    assert np.array_equal(y_b - y0, np.broadcast_to(synth.bf16_to_f32(bias).astype(np.float64), y0.shape))


def test_linear_at_matches_full():
    qa = random_codes((17, 64), 8)
    qw = random_codes((9, 64), 9)
    sa = np.linspace(0.3, 0.9, 17).astype(np.float32)
    sw = np.linspace(0.02, 0.05, 9).astype(np.float32)
    bias = synth.normal_bf16("test/gemm_at_bias", (9,), 0.1)
    y = oracle.linear(qa, sa, qw, sw, bias)
    ms = np.array([0, 16, 3, 7, 16])
    ns = np.array([0, 8, 5, 0, 1])
    assert np.array_equal(oracle.linear_at(qa, sa, qw, sw, bias, ms, ns), y[ms, ns])


def test_tolerance_helper():
    ref = np.array([1.0, -2.0, 0.0, 100.0])
    ok, _ = oracle.tolerance_ok(ref * (1 + 0.009), ref)
    assert ok
    bad, _ = oracle.tolerance_ok(ref * (1 + 0.02), ref)
    assert not bad


def test_weight_only_matches_float64_matmul_and_closed_form():
    """The weight-only oracle against numpy's float64 matmul of the values
    decoded by PyTorch (products exact; sums agree to double rounding), and a
    closed form with constant operands."""
    a = synth.normal_bf16("test/wo/a", (7, 96), 1.5)
    qw = random_codes((5, 96), 11)
    sw = np.linspace(0.5, 2.0, 5).astype(np.float32)
    bias = synth.normal_bf16("test/wo/b", (5,), 0.1)
    y = oracle.linear_weight_only(a, qw, sw, bias)
    av = synth.bf16_to_f32(a).astype(np.float64)
    ref = (av @ torch_decode(qw).T) * sw.astype(np.float64)[None, :] + synth.bf16_to_f32(bias).astype(np.float64)[None, :]
    assert np.allclose(y, ref, rtol=1e-14, atol=1e-12)
    ones = np.full((2, 64), 0x3F80, dtype=np.uint16)  # 1.0
    qc = np.full((3, 64), 0x40, dtype=np.uint8)       # 2.0
    y1 = oracle.linear_weight_only(ones, qc, np.array([1.0, 0.5, 0.25], dtype=np.float32))
    assert np.array_equal(y1, np.array([[128.0, 64.0, 32.0]] * 2))
