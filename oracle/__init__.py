"""CPU oracle for the FP8 DiT linear path — TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package. The product library (``dit_rowwise_amax_b200``)
never imports it and shares no code with it.

What it computes (see oracle.c for the page citations):
  * ``decode`` / ``encode``: OCP E4M3FN and E5M2, round-half-even, saturating.
  * ``quantize_rows``: per-row amax, S = fp32(amax) / fmax, q = encode(x / S).
  * ``quantize_tensor``: the same with one amax per tensor;
    ``quantize_tensor_typed`` for bf16, fp16 or fp32 tensors.
  * ``linear``: exact integer dot of dequantised E4M3 operands, then
    y = dot * sa[m] * sw[n] + bias[n] in double.
  * ``linear_weight_only``: bf16 activation x decoded E4M3 weight, per-channel
    scale and bias, in double.
  * ``act_bf16``: the producer activation (GELU erf / tanh form, SiLU) in
    double, rounded once to bf16.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

E4M3FN = 0
E5M2 = 1
FMAX = {E4M3FN: 448.0, E5M2: 57344.0}

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

_p = ctypes.c_void_p
_i64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, OpenMP, no fast-math)."""
    src = os.path.join(_HERE, "oracle.c")
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
                               "-ffp-contract=off", src, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        lib.or_decode.restype = ctypes.c_double
        lib.or_decode.argtypes = [ctypes.c_int, ctypes.c_uint8]
        lib.or_encode.restype = ctypes.c_uint8
        lib.or_encode.argtypes = [ctypes.c_int, ctypes.c_float]
        lib.or_encode_many.restype = None
        lib.or_encode_many.argtypes = [ctypes.c_int, _p, _i64, _p]
        lib.or_quantize_rows.restype = None
        lib.or_quantize_rows.argtypes = [_p, _i64, _i64, _i64, ctypes.c_int, _p, _i64, _p]
        lib.or_quantize_tensor.restype = None
        lib.or_quantize_tensor.argtypes = [_p, _i64, ctypes.c_int, _p, _p]
        lib.or_quantize_tensor_typed.restype = None
        lib.or_quantize_tensor_typed.argtypes = [_p, ctypes.c_int, _i64, ctypes.c_int, _p, _p]
        lib.or_f16_to_f32.restype = ctypes.c_float
        lib.or_f16_to_f32.argtypes = [ctypes.c_uint16]
        lib.or_linear.restype = None
        lib.or_linear.argtypes = [_p, _p, _p, _p, _p, _i64, _i64, _i64, _p]
        lib.or_linear_at.restype = None
        lib.or_linear_at.argtypes = [_p, _p, _p, _p, _p, _i64, _p, _p, _i64, _p]
        lib.or_linear_weight_only.restype = None
        lib.or_linear_weight_only.argtypes = [_p, _p, _p, _p, _i64, _i64, _i64, _p]
        lib.or_act.restype = ctypes.c_double
        lib.or_act.argtypes = [ctypes.c_int, ctypes.c_double]
        lib.or_round_bf16.restype = ctypes.c_uint16
        lib.or_round_bf16.argtypes = [ctypes.c_double]
        lib.or_act_bf16.restype = None
        lib.or_act_bf16.argtypes = [ctypes.c_int, _p, _i64, _p]
        lib.or_num_threads.restype = ctypes.c_int
        lib.or_num_threads.argtypes = []
        lib.or_set_threads.restype = None
        lib.or_set_threads.argtypes = [ctypes.c_int]
        lib.or_dot_units.restype = None
        lib.or_dot_units.argtypes = [_p, _p, _i64, _i64, _i64, _p]
        _lib = lib
    return _lib


def _c(a: np.ndarray, dtype) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == dtype, (a.dtype, dtype)
    return a


def decode(fmt: int, code: int) -> float:
    return float(_load().or_decode(fmt, code))


def decode_table(fmt: int) -> np.ndarray:
    return np.array([decode(fmt, c) for c in range(256)], dtype=np.float64)


def encode(fmt: int, v: np.ndarray) -> np.ndarray:
    v = _c(np.asarray(v, dtype=np.float32), np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    _load().or_encode_many(fmt, v.ctypes.data, v.size, out.ctypes.data)
    return out


def quantize_rows(x: np.ndarray, fmt: int = E4M3FN):
    """x: uint16 bf16 patterns [M, K] -> (q uint8 [M, K], s float32 [M])."""
    x = _c(x, np.uint16)
    M, K = x.shape
    q = np.empty((M, K), dtype=np.uint8)
    s = np.empty((M,), dtype=np.float32)
    _load().or_quantize_rows(x.ctypes.data, M, K, K, fmt, q.ctypes.data, K, s.ctypes.data)
    return q, s


def quantize_tensor(x: np.ndarray, fmt: int):
    """x: uint16 bf16 patterns, any shape -> (q uint8 same shape, s float32 scalar)."""
    x = _c(x, np.uint16)
    q = np.empty(x.shape, dtype=np.uint8)
    s = np.empty((1,), dtype=np.float32)
    _load().or_quantize_tensor(x.ctypes.data, x.size, fmt, q.ctypes.data, s.ctypes.data)
    return q, float(s[0])


SRC_BF16, SRC_F16, SRC_F32 = 0, 1, 2


def quantize_tensor_typed(x: np.ndarray, fmt: int):
    """Per-tensor quantisation of a bf16 (uint16 patterns), float16 or float32
    array, any shape -> (q uint8 same shape, s float32 scalar)."""
    src = {np.dtype(np.uint16): SRC_BF16, np.dtype(np.float16): SRC_F16, np.dtype(np.float32): SRC_F32}[x.dtype]
    x = np.ascontiguousarray(x)
    q = np.empty(x.shape, dtype=np.uint8)
    s = np.empty((1,), dtype=np.float32)
    _load().or_quantize_tensor_typed(x.ctypes.data, src, x.size, fmt, q.ctypes.data, s.ctypes.data)
    return q, float(s[0])


def f16_to_f32(bits: int) -> float:
    """The oracle's closed-form decode of one binary16 bit pattern."""
    return float(_load().or_f16_to_f32(bits))


def linear(qa, sa, qw, sw, bias=None) -> np.ndarray:
    """Exact dequantised E4M3 GEMM + epilogue in double: y [M, N] float64."""
    qa, qw = _c(qa, np.uint8), _c(qw, np.uint8)
    sa, sw = _c(sa, np.float32), _c(sw, np.float32)
    M, K = qa.shape
    N = qw.shape[0]
    assert qw.shape[1] == K and sa.shape == (M,) and sw.shape == (N,)
    b = None if bias is None else _c(bias, np.uint16)
    y = np.empty((M, N), dtype=np.float64)
    _load().or_linear(qa.ctypes.data, sa.ctypes.data, qw.ctypes.data, sw.ctypes.data,
                      None if b is None else b.ctypes.data, M, N, K, y.ctypes.data)
    return y


def linear_weight_only(a, qw, sw, bias=None) -> np.ndarray:
    """bf16 activation x E4M3 weight (decoded), per-channel scale, bias, in double."""
    a, qw, sw = _c(a, np.uint16), _c(qw, np.uint8), _c(sw, np.float32)
    M, K = a.shape
    N = qw.shape[0]
    assert qw.shape[1] == K and sw.shape == (N,)
    b = None if bias is None else _c(bias, np.uint16)
    y = np.empty((M, N), dtype=np.float64)
    _load().or_linear_weight_only(a.ctypes.data, qw.ctypes.data, sw.ctypes.data,
                                  None if b is None else b.ctypes.data, M, N, K, y.ctypes.data)
    return y


def linear_at(qa, sa, qw, sw, bias, ms, ns) -> np.ndarray:
    """The oracle linear at listed (ms[i], ns[i]) positions only."""
    qa, qw = _c(qa, np.uint8), _c(qw, np.uint8)
    sa, sw = _c(sa, np.float32), _c(sw, np.float32)
    ms, ns = _c(np.asarray(ms, dtype=np.int64), np.int64), _c(np.asarray(ns, dtype=np.int64), np.int64)
    K = qa.shape[1]
    b = None if bias is None else _c(bias, np.uint16)
    y = np.empty(ms.shape, dtype=np.float64)
    _load().or_linear_at(qa.ctypes.data, sa.ctypes.data, qw.ctypes.data, sw.ctypes.data,
                         None if b is None else b.ctypes.data, K, ms.ctypes.data, ns.ctypes.data,
                         ms.size, y.ctypes.data)
    return y


def dot_units(qa, qw) -> np.ndarray:
    """Integer dots sum_k u(A[m,k]) u(W[n,k]), u(code) = value * 2^9 (int64 [M, N])."""
    qa, qw = _c(qa, np.uint8), _c(qw, np.uint8)
    M, K = qa.shape
    N = qw.shape[0]
    out = np.empty((M, N), dtype=np.int64)
    _load().or_dot_units(qa.ctypes.data, qw.ctypes.data, M, N, K, out.ctypes.data)
    return out


ACT_GELU_ERF = 1
ACT_GELU_TANH = 2
ACT_SILU = 3


def act(kind: int, x: float) -> float:
    """The producer activation in double."""
    return float(_load().or_act(kind, x))


def round_bf16(v: float) -> int:
    """Nearest bf16 bit pattern to a double (ties to even)."""
    return int(_load().or_round_bf16(v))


def act_bf16(kind: int, h: np.ndarray) -> np.ndarray:
    """bf16(act(h)) elementwise; h and the result are uint16 bf16 patterns."""
    h = _c(h, np.uint16)
    g = np.empty(h.shape, dtype=np.uint16)
    _load().or_act_bf16(kind, h.ctypes.data, h.size, g.ctypes.data)
    return g


def num_threads() -> int:
    """Threads the oracle's OpenMP loops use."""
    return int(_load().or_num_threads())


def set_threads(n: int) -> None:
    """Threads for the oracle's loops from now on; n <= 0 restores the default."""
    _load().or_set_threads(int(n))


def tolerance_ok(gpu: np.ndarray, ref: np.ndarray, rms_ref: float | None = None):
    """|gpu - ref| <= 1e-2 |ref| + 1e-3 rms(ref), elementwise. Returns (ok, worst ratio)."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if rms_ref is None:
        rms_ref = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    bound = 1e-2 * np.abs(ref) + 1e-3 * rms_ref
    err = np.abs(gpu - ref)
    ratio = float(np.max(err / np.maximum(bound, 1e-300))) if ref.size else 0.0
    return bool(np.all(err <= bound)), ratio
