"""Seeded synthetic inputs for the FP8 DiT linear workloads.

The shapes and value distributions follow the workloads of
"从 BF16 到 FP8：HunyuanVideo1.5推理优化复盘" (sections 三.2 and 三.4: FFN up
M=4096 N=8192 K=2048, FFN down M=4096 N=2048 K=8192, hidden_states
[1, 32760, 2048] and encoder_hidden_states [1, 26, 2048] through Q/K/V) and
the state-dict conversion of "Quantize Model to FP8 Format". The pages give
shapes, not data, so every tensor is drawn here from a counter-based stream
(see synth.c); both the CPU oracle and the CUDA path read these same bytes.

Arrays are numpy uint16 holding bf16 bit patterns. Nothing here quantises.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libsynth.so")
_lib = None

SEED = 0


def build(force: bool = False) -> str:
    """Compile synth.c into libsynth.so beside it (gcc, OpenMP)."""
    src = os.path.join(_HERE, "synth.c")
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
        lib.synth_key.restype = ctypes.c_uint64
        lib.synth_key.argtypes = [ctypes.c_uint64, ctypes.c_char_p]
        lib.synth_normal_bf16.restype = None
        lib.synth_normal_bf16.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_double,
                                          ctypes.c_double, ctypes.c_double, ctypes.c_double,
                                          ctypes.c_void_p]
        lib.synth_gelu_normal_bf16.restype = None
        lib.synth_gelu_normal_bf16.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p]
        lib.synth_uniform.restype = None
        lib.synth_uniform.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p]
        _lib = lib
    return _lib


def key(name: str, seed: int = SEED) -> int:
    return int(_load().synth_key(seed, name.encode()))


def normal_bf16(name: str, shape, std: float = 1.0, mean: float = 0.0,
                outlier_p: float = 0.0, outlier_factor: float = 1.0, seed: int = SEED,
                out: np.ndarray | None = None) -> np.ndarray:
    n = int(np.prod(shape))
    if out is None:
        out = np.empty(shape, dtype=np.uint16)
    assert out.dtype == np.uint16 and out.flags.c_contiguous and out.size == n
    _load().synth_normal_bf16(key(name, seed), n, mean, std, outlier_p, outlier_factor,
                              out.ctypes.data)
    return out


def gelu_normal_bf16(name: str, shape, seed: int = SEED) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(shape, dtype=np.uint16)
    _load().synth_gelu_normal_bf16(key(name, seed), n, out.ctypes.data)
    return out


def uniform(name: str, n: int, seed: int = SEED) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    _load().synth_uniform(key(name, seed), n, out.ctypes.data)
    return out


def bf16_to_f32(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float32."""
    return (a.astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------- workloads
@dataclass(frozen=True)
class LinearShape:
    name: str
    M: int
    N: int
    K: int


TINY = LinearShape("tiny", 64, 512, 256)
FFN_UP = LinearShape("ffn_up", 4096, 8192, 2048)
FFN_DOWN = LinearShape("ffn_down", 4096, 2048, 8192)
ATTN_HIDDEN_M = 32760
ATTN_ENCODER_M = 26
ATTN_D = 2048


def tiny(seed: int = SEED) -> dict:
    """A[64,256] ~N(0,1) with 1% of entries x20, W[512,256] ~N(0,0.02), bias[512] ~N(0,0.1)."""
    s = TINY
    return {
        "A": normal_bf16("tiny/A", (s.M, s.K), 1.0, outlier_p=0.01, outlier_factor=20.0, seed=seed),
        "W": normal_bf16("tiny/W", (s.N, s.K), 0.02, seed=seed),
        "bias": normal_bf16("tiny/bias", (s.N,), 0.1, seed=seed),
    }


def ffn_up(seed: int = SEED) -> dict:
    """A[4096,2048] ~N(0,1) with 0.5% x30 outliers, W[8192,2048] ~N(0,0.02), bias[8192] ~N(0,0.1)."""
    s = FFN_UP
    return {
        "A": normal_bf16("ffn_up/A", (s.M, s.K), 1.0, outlier_p=0.005, outlier_factor=30.0, seed=seed),
        "W": normal_bf16("ffn_up/W", (s.N, s.K), 0.02, seed=seed),
        "bias": normal_bf16("ffn_up/bias", (s.N,), 0.1, seed=seed),
    }


def ffn_down(seed: int = SEED) -> dict:
    """A[4096,8192] = GELU(N(0,1)), W[2048,8192] ~N(0,0.015), bias[2048] ~N(0,0.1)."""
    s = FFN_DOWN
    return {
        "A": gelu_normal_bf16("ffn_down/A", (s.M, s.K), seed=seed),
        "W": normal_bf16("ffn_down/W", (s.N, s.K), 0.015, seed=seed),
        "bias": normal_bf16("ffn_down/bias", (s.N,), 0.1, seed=seed),
    }


def attention(seed: int = SEED, hidden_rows: int = ATTN_HIDDEN_M) -> dict:
    """hidden[32760,2048] ~N(0,1), encoder[26,2048] ~N(0,1), W_q/W_k/W_v [2048,2048] ~N(0,0.02),
    bias_q/k/v [2048] ~N(0,0.1). ``hidden_rows`` takes the first rows of the same stream."""
    d = ATTN_D
    out = {
        "hidden": normal_bf16("attention/hidden", (ATTN_HIDDEN_M, d), 1.0, seed=seed)[:hidden_rows].copy(),
        "encoder": normal_bf16("attention/encoder", (ATTN_ENCODER_M, d), 1.0, seed=seed),
    }
    for p in ("q", "k", "v"):
        out[f"W_{p}"] = normal_bf16(f"attention/W_{p}", (d, d), 0.02, seed=seed)
        out[f"bias_{p}"] = normal_bf16(f"attention/bias_{p}", (d,), 0.1, seed=seed)
    return out


STATE_DICT_BLOCKS = 32
STATE_DICT_BLOCK_SHAPES = (
    ("attn.to_q.weight", (2048, 2048)),
    ("attn.to_k.weight", (2048, 2048)),
    ("attn.to_v.weight", (2048, 2048)),
    ("attn.to_out.weight", (2048, 2048)),
    ("ffn.up.weight", (8192, 2048)),
    ("ffn.down.weight", (2048, 8192)),
)


def state_dict_layout(blocks: int = STATE_DICT_BLOCKS):
    """[(name, shape)] of the synthetic DiT weight set: 32 blocks x 6 tensors."""
    return [(f"blocks.{b}.{n}", shp) for b in range(blocks) for n, shp in STATE_DICT_BLOCK_SHAPES]


def state_dict_tensor(name: str, shape, seed: int = SEED, out: np.ndarray | None = None) -> np.ndarray:
    """One tensor of the weight set: ~N(0,0.02) with 1e-3 of entries x50."""
    return normal_bf16("state_dict/" + name, shape, 0.02, outlier_p=1e-3, outlier_factor=50.0,
                       seed=seed, out=out)
