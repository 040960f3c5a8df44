"""fp8dit: FP8 linear layer of a diffusion / video DiT on B200 (sm_100a).

Thin Python binding over the C-ABI library ``libfp8dit.so`` (declared in
``include/fp8dit.h``). This module only marshals arguments: it checks
tensors, allocates outputs with torch, and passes device pointers and the
current CUDA stream to the library. Every step of the path (amax,
quantisation, GEMM, epilogue, conversion) runs in the library's kernels.
There is no fallback: if the library is missing or a call fails, an
exception is raised.

Path ("从 BF16 到 FP8：HunyuanVideo1.5推理优化复盘", section 三.1):
BF16 activation -> dynamic per-token E4M3 quantisation -> FP8 GEMM against
per-channel pre-quantised, K-major E4M3 weights -> scale / bias / bf16.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, List, Optional, Sequence, Tuple

import torch

__all__ = [
    "E4M3FN", "E5M2", "Fp8DitError", "FP8Linear", "library_path", "load_library",
    "quantize_rowwise", "act_quantize_rowwise", "quantize_weight_per_channel", "quantize_per_tensor", "convert_state_dict",
    "scaled_linear_multi", "device_error", "selftest_expired_wait", "selftest_quotient", "as_float8",
]

E4M3FN = 0
E5M2 = 1
_FORMAT_NAMES = {"float8_e4m3fn": E4M3FN, "e4m3fn": E4M3FN, "e4m3": E4M3FN,
                 "float8_e5m2": E5M2, "e5m2": E5M2, E4M3FN: E4M3FN, E5M2: E5M2}
_TORCH_FP8 = {E4M3FN: torch.float8_e4m3fn, E5M2: torch.float8_e5m2}

_STATUS = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED_SHAPE", 3: "EMPTY", 4: "CUDA", 5: "TIMEOUT"}

_PKG = os.path.dirname(os.path.abspath(__file__))
_lib = None


class Fp8DitError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"fp8dit {_STATUS.get(status, status)}: {message}")
        self.status = status


def library_path() -> str:
    return os.path.join(_PKG, "libfp8dit.so")


class _TensorDesc(ctypes.Structure):
    _fields_ = [("src", ctypes.c_void_p), ("numel", ctypes.c_int64), ("dst", ctypes.c_void_p),
                ("scale", ctypes.c_void_p), ("src_dtype", ctypes.c_int32), ("reserved", ctypes.c_int32)]


# Source element types of the per-tensor conversion (fp8dit_src_dtype).
_SRC_DTYPES = {torch.bfloat16: 0, torch.float16: 1, torch.float32: 2}
_FP8_DTYPES = (torch.float8_e4m3fn, torch.float8_e5m2)


def load_library():
    """Load libfp8dit.so; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m dit_rowwise_amax_b200.build`")
    L = ctypes.CDLL(path)
    p, i64, i32, st = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int
    L.fp8_quantize_rowwise.argtypes = [p, i64, i64, i64, ctypes.c_int, p, i64, p, p]
    L.fp8_quantize_weight_per_channel.argtypes = [p, i64, i64, ctypes.c_int, p, p, p]
    L.fp8_act_quantize_rowwise.argtypes = [p, i64, i64, i64, ctypes.c_int, p, i64, p, p, i64, p]
    L.fp8_quantize_weight_per_tensor_workspace_size.argtypes = [i32]
    L.fp8_quantize_weight_per_tensor_workspace_size.restype = ctypes.c_size_t
    L.fp8_quantize_weight_per_tensor.argtypes = [ctypes.POINTER(_TensorDesc), i32, ctypes.c_int, p,
                                                 ctypes.c_size_t, p]
    L.fp8_linear_create.argtypes = [i64, i64, p, p, p, ctypes.c_int, ctypes.POINTER(p)]
    L.fp8_linear_destroy.argtypes = [p]
    L.fp8_linear_workspace_size.argtypes = [p]
    L.fp8_linear_workspace_size.restype = ctypes.c_size_t
    L.fp8_linear_set_workspace.argtypes = [p, p, ctypes.c_size_t]
    L.fp8_linear_workspace_flag_bytes.argtypes = [p]
    L.fp8_linear_workspace_flag_bytes.restype = ctypes.c_size_t
    L.fp8_scaled_linear.argtypes = [p, i64, p, p, p, p, p, p, p]
    L.fp8_scaled_linear_multi.argtypes = [ctypes.POINTER(p), i32, i64, p, p, p, ctypes.POINTER(p), p]
    L.fp8_scaled_linear_noalloc.argtypes = [p, i64, p, p, p]
    L.fp8_weight_only_linear.argtypes = [p, i64, p, p, p]
    L.fp8_scaled_linear_fused.argtypes = [p, i64, p, p, p, p, p]
    L.fp8_linear_host_workspace_size.argtypes = [p, i64, i32]
    L.fp8_linear_host_workspace_size.restype = ctypes.c_size_t
    L.fp8_linear_set_host_pipeline.argtypes = [p, p, ctypes.c_size_t, i64, i32]
    L.fp8_scaled_linear_host.argtypes = [p, i64, p, p, p]
    L.fp8_linear_plan.argtypes = [p, i64, i32, ctypes.POINTER(i32), ctypes.POINTER(i32), ctypes.POINTER(i32)]
    L.fp8dit_device_error.argtypes = [p]
    L.fp8dit_selftest_expired_wait.argtypes = [i64, p]
    L.fp8dit_selftest_quotient.argtypes = [p, p]
    L.fp8dit_last_error_string.restype = ctypes.c_char_p
    for name in ("fp8_quantize_rowwise", "fp8_act_quantize_rowwise", "fp8_quantize_weight_per_channel",
                 "fp8_quantize_weight_per_tensor",
                 "fp8_linear_create", "fp8_linear_destroy", "fp8_scaled_linear", "fp8_scaled_linear_multi",
                 "fp8_scaled_linear_noalloc", "fp8_weight_only_linear", "fp8_scaled_linear_fused",
                 "fp8_linear_set_host_pipeline", "fp8_scaled_linear_host",
                 "fp8_linear_plan", "fp8_linear_set_workspace", "fp8dit_device_error",
                 "fp8dit_selftest_expired_wait",
                 "fp8dit_selftest_quotient"):
        getattr(L, name).restype = st
    _lib = L
    return L


def _check(status: int):
    if status != 0:
        msg = load_library().fp8dit_last_error_string().decode(errors="replace")
        raise Fp8DitError(status, msg)


def _stream(device: torch.device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _fmt(fmt) -> int:
    try:
        return _FORMAT_NAMES[fmt]
    except KeyError:
        raise ValueError(f"unknown FP8 format {fmt!r}") from None


def _bf16_matrix(x: torch.Tensor, name: str) -> torch.Tensor:
    if not x.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if x.dtype not in (torch.bfloat16, torch.int16, torch.uint16):
        raise ValueError(f"{name} must hold bf16 values (got {x.dtype})")
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError(f"{name} must be a 2-D tensor with contiguous rows")
    return x


_CODE_DTYPES = (torch.uint8, torch.float8_e4m3fn, torch.float8_e5m2)
_BF16_DTYPES = (torch.bfloat16, torch.int16, torch.uint16)


def _check_out(t: torch.Tensor, name: str, dtypes, shape, device: torch.device, rows_only: bool = False):
    """A caller-supplied output or scratch tensor: the library writes through
    its data pointer, so dtype, shape and device must be exactly right.
    rows_only: only the last dimension needs to be contiguous (row stride free)."""
    ok = (isinstance(t, torch.Tensor) and t.dtype in dtypes and tuple(t.shape) == tuple(shape)
          and t.device == device and (t.stride(-1) == 1 if rows_only else t.is_contiguous()))
    if not ok:
        names = "/".join(str(d).replace("torch.", "") for d in dtypes)
        raise ValueError(f"{name} must be a {'row-contiguous' if rows_only else 'contiguous'} {names} tensor "
                         f"of shape {tuple(shape)} on {device}")
    return t


def _same_device(t: torch.Tensor, device: torch.device, name: str):
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, the layer on {device}")


def as_float8(q: torch.Tensor, fmt=E4M3FN) -> torch.Tensor:
    """View raw FP8 codes (uint8) as torch's float8 dtype of the format."""
    return q.view(_TORCH_FP8[_fmt(fmt)])


def quantize_rowwise(x: torch.Tensor, fmt=E4M3FN, q: Optional[torch.Tensor] = None,
                     scale: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Per-token amax quantisation of bf16 x [M, K] -> (codes uint8 [M, K], S float32 [M])."""
    x = _bf16_matrix(x, "x")
    M, K = x.shape
    if q is None:
        q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    if scale is None:
        scale = torch.empty((M,), dtype=torch.float32, device=x.device)
    _check_out(q, "q", _CODE_DTYPES, (M, K), x.device, rows_only=True)
    _check_out(scale, "scale", (torch.float32,), (M,), x.device)
    _check(load_library().fp8_quantize_rowwise(x.data_ptr(), M, K, x.stride(0), _fmt(fmt), q.data_ptr(),
                                               q.stride(0), scale.data_ptr(), _stream(x.device)))
    return q, scale


ACTIVATIONS = {"gelu": 1, "gelu_erf": 1, "gelu_tanh": 2, "silu": 3}


def act_quantize_rowwise(h: torch.Tensor, act: str = "gelu", q: Optional[torch.Tensor] = None,
                         scale: Optional[torch.Tensor] = None, return_bf16: bool = False):
    """Producer fusion: bf16(act(h)) quantised per token to E4M3FN in one pass.
    Returns (codes uint8 [M, K], S float32 [M]) and, with return_bf16, the bf16 activation."""
    h = _bf16_matrix(h, "h")
    M, K = h.shape
    if q is None:
        q = torch.empty((M, K), dtype=torch.uint8, device=h.device)
    if scale is None:
        scale = torch.empty((M,), dtype=torch.float32, device=h.device)
    _check_out(q, "q", _CODE_DTYPES, (M, K), h.device, rows_only=True)
    _check_out(scale, "scale", (torch.float32,), (M,), h.device)
    g = torch.empty((M, K), dtype=torch.bfloat16, device=h.device) if return_bf16 else None
    try:
        kind = ACTIVATIONS[act]
    except KeyError:
        raise ValueError(f"unknown activation {act!r}") from None
    _check(load_library().fp8_act_quantize_rowwise(h.data_ptr(), M, K, h.stride(0), kind, q.data_ptr(), q.stride(0),
                                                   scale.data_ptr(), None if g is None else g.data_ptr(),
                                                   K if g is not None else 0, _stream(h.device)))
    return (q, scale, g) if return_bf16 else (q, scale)


def quantize_weight_per_channel(w: torch.Tensor, fmt=E4M3FN) -> Tuple[torch.Tensor, torch.Tensor]:
    """Per-output-channel quantisation of bf16 W [N, K] -> K-major codes [N, K] and S [N]."""
    w = _bf16_matrix(w, "w")
    if not w.is_contiguous():
        raise ValueError("w must be contiguous")
    N, K = w.shape
    qw = torch.empty((N, K), dtype=torch.uint8, device=w.device)
    sw = torch.empty((N,), dtype=torch.float32, device=w.device)
    _check(load_library().fp8_quantize_weight_per_channel(w.data_ptr(), N, K, _fmt(fmt), qw.data_ptr(),
                                                          sw.data_ptr(), _stream(w.device)))
    return qw, sw


def _src_dtype(t: torch.Tensor) -> int:
    if t.dtype in (torch.int16, torch.uint16):  # raw bf16 bit patterns
        return 0
    try:
        return _SRC_DTYPES[t.dtype]
    except KeyError:
        raise ValueError(f"tensors must be bfloat16, float16 or float32 (got {t.dtype})") from None


def quantize_per_tensor(tensors: Sequence[torch.Tensor], fmt=E5M2,
                        outs: Optional[Sequence[torch.Tensor]] = None,
                        scales: Optional[torch.Tensor] = None,
                        workspace: Optional[torch.Tensor] = None) -> Tuple[List[torch.Tensor], torch.Tensor]:
    """Per-tensor amax conversion of bf16 / fp16 / fp32 tensors (dtypes may be
    mixed) -> (codes uint8 per tensor, S float32 [n])."""
    L = load_library()
    n = len(tensors)
    if n == 0:
        _check(L.fp8_quantize_weight_per_tensor(None, 0, _fmt(fmt), None, 0, None))
    dev = tensors[0].device
    for t in tensors:
        if not t.is_cuda or t.device != dev or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors on one device")
        _src_dtype(t)
    if outs is None:
        outs = [torch.empty(t.shape, dtype=torch.uint8, device=dev) for t in tensors]
    if scales is None:
        scales = torch.ones((n,), dtype=torch.float32, device=dev)
    if len(outs) != n:
        raise ValueError("outs must hold one tensor per input tensor")
    for i, (t, o) in enumerate(zip(tensors, outs)):
        _check_out(o, f"outs[{i}]", _CODE_DTYPES, t.shape, dev)
    _check_out(scales, "scales", (torch.float32,), (n,), dev)
    ws_bytes = int(L.fp8_quantize_weight_per_tensor_workspace_size(n))
    if workspace is None:
        workspace = torch.empty((ws_bytes,), dtype=torch.uint8, device=dev)
    if workspace.device != dev or not workspace.is_contiguous() or workspace.numel() * workspace.element_size() < ws_bytes:
        raise ValueError(f"workspace must be a contiguous tensor of at least {ws_bytes} bytes on {dev}")
    descs = (_TensorDesc * n)()
    for i, (t, o) in enumerate(zip(tensors, outs)):
        descs[i].src, descs[i].numel, descs[i].dst = t.data_ptr(), t.numel(), o.data_ptr()
        descs[i].scale = scales.data_ptr() + 4 * i
        descs[i].src_dtype, descs[i].reserved = _src_dtype(t), 0
    _check(L.fp8_quantize_weight_per_tensor(descs, n, _fmt(fmt), workspace.data_ptr(),
                                            workspace.numel() * workspace.element_size(), _stream(dev)))
    return list(outs), scales


def convert_state_dict(state_dict, fp8_format: str = "float8_e5m2"):
    """Convert a state-dict's floating tensors to FP8 with one amax scale each
    ("Quantize Model to FP8 Format": model_state_dict + fp8_format, default
    float8_e5m2). Returns (quantised dict, {name: fp32 scale tensor}).

    bfloat16, float16 and float32 tensors with numel > 0 are converted, in one
    launch whatever the mix of dtypes; they must be on a CUDA device (there is
    no CPU path). Non-floating entries, empty tensors and tensors that are
    already FP8 pass through unchanged. Any other floating dtype (float64)
    raises ValueError rather than passing through unconverted. Raises
    ValueError("Invalid input.") for a non-dict or empty dict, and Fp8DitError
    (EMPTY) when no tensor was converted.
    """
    if not isinstance(state_dict, dict) or len(state_dict) == 0:
        raise ValueError("Invalid input.")
    fmt = _fmt(fp8_format)
    names = []
    for k, v in state_dict.items():
        if not isinstance(v, torch.Tensor) or not v.is_floating_point() or v.dtype in _FP8_DTYPES or v.numel() == 0:
            continue
        if v.dtype not in _SRC_DTYPES:
            raise ValueError(f"{k}: {v.dtype} is not convertible (bfloat16, float16 or float32)")
        if not v.is_cuda:
            raise ValueError(f"{k}: floating tensors must be on a CUDA device to be converted")
        names.append(k)
    if not names:
        raise Fp8DitError(3, f"No tensor converted to {fp8_format}.")
    tensors = [state_dict[k].contiguous() for k in names]
    outs, scales = quantize_per_tensor(tensors, fmt)
    out = dict(state_dict)
    scale_map = {}
    for i, k in enumerate(names):
        out[k] = outs[i].view(_TORCH_FP8[fmt])
        scale_map[k] = scales[i]
    return out, scale_map


class FP8Linear:
    """One FP8 linear layer: y = (A W^T) * sa * sw + bias, bf16 out.

    Construction quantises W per output channel (K-major codes, no transpose)
    and binds the tile plan and weight TMA descriptors once
    ("从 BF16 到 FP8", section 三.3). ``forward`` takes a bf16 activation and
    quantises it per token; ``forward_fp8`` takes an already-quantised
    (codes, per-token scale) pair (section 三.5).
    """

    def __init__(self, qw: torch.Tensor, sw: torch.Tensor, bias: Optional[torch.Tensor] = None):
        if qw.dtype != torch.uint8 or qw.dim() != 2 or not qw.is_contiguous() or not qw.is_cuda:
            raise ValueError("qw must be contiguous uint8 [N, K] on a CUDA device")
        if sw.dtype != torch.float32 or sw.shape != (qw.shape[0],) or not sw.is_contiguous():
            raise ValueError("sw must be contiguous float32 [N]")
        if bias is not None and (bias.dtype not in (torch.bfloat16, torch.int16, torch.uint16)
                                 or bias.shape != (qw.shape[0],) or not bias.is_contiguous()):
            raise ValueError("bias must be contiguous bf16 [N]")
        self.qw, self.sw, self.bias = qw, sw, bias  # the handle borrows these
        self.N, self.K = qw.shape
        self.device = qw.device
        h = ctypes.c_void_p()
        _check(load_library().fp8_linear_create(self.N, self.K, qw.data_ptr(), sw.data_ptr(),
                                                None if bias is None else bias.data_ptr(),
                                                qw.device.index if qw.device.index is not None
                                                else torch.cuda.current_device(), ctypes.byref(h)))
        self._h = h

    @classmethod
    def from_weight(cls, w: torch.Tensor, bias: Optional[torch.Tensor] = None) -> "FP8Linear":
        qw, sw = quantize_weight_per_channel(w, E4M3FN)
        return cls(qw, sw, bias)

    @property
    def handle(self) -> ctypes.c_void_p:
        return self._h

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            load_library().fp8_linear_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def attach_workspace(self, workspace: Optional[torch.Tensor] = None) -> Optional[torch.Tensor]:
        """Attach a workspace (allocated here when not given) and return it,
        so that it can be attached to further layers whose calls run one after
        another. It enables the stream-K schedule (a nearly empty last wave of
        pair tiles) and split-K (few rows and a long K, FP8 and weight-only);
        detach_workspace() goes back to the plain schedule. Attach only while
        no call of the layer is in flight."""
        L = load_library()
        need = int(L.fp8_linear_workspace_size(self._h))
        if workspace is None:
            workspace = torch.empty((need,), dtype=torch.uint8, device=self.device)
        if workspace.numel() * workspace.element_size() < need or not workspace.is_cuda:
            raise ValueError(f"workspace must be a CUDA tensor of at least {need} bytes")
        _check(L.fp8_linear_set_workspace(self._h, workspace.data_ptr(), workspace.numel() * workspace.element_size()))
        self.workspace = workspace  # keep it alive while attached
        return workspace

    def workspace_flag_bytes(self) -> int:
        """Bytes at the start of the workspace holding flags and counters (zero
        after attaching and between launches)."""
        return int(load_library().fp8_linear_workspace_flag_bytes(self._h))

    def detach_workspace(self) -> None:
        _check(load_library().fp8_linear_set_workspace(self._h, None, 0))
        self.workspace = None

    def plan(self, M: int, n_problems: int = 1) -> Tuple[int, int, int]:
        bm, bn, ctas = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
        _check(load_library().fp8_linear_plan(self._h, M, n_problems, ctypes.byref(bm), ctypes.byref(bn),
                                              ctypes.byref(ctas)))
        return bm.value, bn.value, ctas.value

    def __call__(self, a: torch.Tensor, **kwargs) -> torch.Tensor:
        """layer(a) is layer.forward(a): quantise + FP8 GEMM + epilogue."""
        return self.forward(a, **kwargs)

    def forward(self, a: torch.Tensor, y: Optional[torch.Tensor] = None,
                qa_scratch: Optional[torch.Tensor] = None,
                sa_scratch: Optional[torch.Tensor] = None) -> torch.Tensor:
        a = _bf16_matrix(a, "a")
        if not a.is_contiguous() or a.shape[1] != self.K:
            raise ValueError(f"a must be contiguous [M, {self.K}]")
        M = a.shape[0]
        _same_device(a, self.device, "a")
        if y is None:
            y = torch.empty((M, self.N), dtype=torch.bfloat16, device=a.device)
        if qa_scratch is None:
            qa_scratch = torch.empty((M, self.K), dtype=torch.uint8, device=a.device)
        if sa_scratch is None:
            sa_scratch = torch.empty((M,), dtype=torch.float32, device=a.device)
        _check_out(y, "y", _BF16_DTYPES, (M, self.N), a.device)
        _check_out(qa_scratch, "qa_scratch", _CODE_DTYPES, (M, self.K), a.device)
        _check_out(sa_scratch, "sa_scratch", (torch.float32,), (M,), a.device)
        _check(load_library().fp8_scaled_linear(self._h, M, a.data_ptr(), None, None, qa_scratch.data_ptr(),
                                                sa_scratch.data_ptr(), y.data_ptr(), _stream(a.device)))
        return y

    __call__ = forward

    def forward_weight_only(self, a: torch.Tensor, y: Optional[torch.Tensor] = None) -> torch.Tensor:
        """FP8 weight-only: bf16 activation (not quantised) x this layer's E4M3
        weight decoded to bf16, on the BF16 tensor cores."""
        a = _bf16_matrix(a, "a")
        if not a.is_contiguous() or a.shape[1] != self.K:
            raise ValueError(f"a must be contiguous [M, {self.K}]")
        M = a.shape[0]
        _same_device(a, self.device, "a")
        if y is None:
            y = torch.empty((M, self.N), dtype=torch.bfloat16, device=a.device)
        _check_out(y, "y", _BF16_DTYPES, (M, self.N), a.device)
        _check(load_library().fp8_weight_only_linear(self._h, M, a.data_ptr(), y.data_ptr(), _stream(a.device)))
        return y

    def forward_fused(self, a: torch.Tensor, y: Optional[torch.Tensor] = None,
                      qa_scratch: Optional[torch.Tensor] = None,
                      sa_scratch: Optional[torch.Tensor] = None) -> torch.Tensor:
        """The FP8 linear from a bf16 activation in one launch: the launch's
        CTAs quantise A per token (each element once) into qa_scratch /
        sa_scratch, then run the GEMM, each tile starting once its rows are
        quantised. Same codes, scales and (with 256 x 256 pair tiles) output
        bits as forward(). Needs a workspace for its counters: one is attached
        here if the layer has none (which also lets forward() use the stream-K
        and split-K schedules)."""
        a = _bf16_matrix(a, "a")
        if not a.is_contiguous() or a.shape[1] != self.K:
            raise ValueError(f"a must be contiguous [M, {self.K}]")
        M = a.shape[0]
        _same_device(a, self.device, "a")
        if getattr(self, "workspace", None) is None:
            self.attach_workspace()
        if y is None:
            y = torch.empty((M, self.N), dtype=torch.bfloat16, device=a.device)
        if qa_scratch is None:
            qa_scratch = torch.empty((M, self.K), dtype=torch.uint8, device=a.device)
        if sa_scratch is None:
            sa_scratch = torch.empty((M,), dtype=torch.float32, device=a.device)
        _check_out(y, "y", _BF16_DTYPES, (M, self.N), a.device)
        _check_out(qa_scratch, "qa_scratch", _CODE_DTYPES, (M, self.K), a.device)
        _check_out(sa_scratch, "sa_scratch", (torch.float32,), (M,), a.device)
        _check(load_library().fp8_scaled_linear_fused(self._h, M, a.data_ptr(), qa_scratch.data_ptr(),
                                                      sa_scratch.data_ptr(), y.data_ptr(), _stream(a.device)))
        return y

    def attach_host_pipeline(self, chunk_rows: int = 2048, slots: int = 2) -> torch.Tensor:
        """Allocate and attach the device workspace of the host-buffer pipeline
        (forward_host); returns it."""
        L = load_library()
        need = int(L.fp8_linear_host_workspace_size(self._h, chunk_rows, slots))
        if need == 0:
            raise ValueError("chunk_rows must be > 0 and slots in 2..8")
        ws = torch.empty((need,), dtype=torch.uint8, device=self.device)
        _check(L.fp8_linear_set_host_pipeline(self._h, ws.data_ptr(), need, chunk_rows, slots))
        self.host_workspace = ws  # keep it alive while attached
        return ws

    def detach_host_pipeline(self) -> None:
        _check(load_library().fp8_linear_set_host_pipeline(self._h, None, 0, 0, 0))
        self.host_workspace = None

    def forward_host(self, a: torch.Tensor, y: Optional[torch.Tensor] = None) -> torch.Tensor:
        """The FP8 linear of a HOST bf16 activation into a HOST bf16 output,
        chunks of rows pipelined through copy-in, quantise + GEMM and copy-out
        (pinned tensors let the copies overlap). Asynchronous on the current
        stream: the result is in ``y`` once that stream has been synchronised,
        and ``a`` must stay unchanged until then."""
        if a.dtype != torch.bfloat16 or a.dim() != 2 or not a.is_contiguous() or a.is_cuda:
            raise ValueError("a must be a contiguous host bf16 [M, K] tensor")
        if a.shape[1] != self.K:
            raise ValueError(f"a must be [M, {self.K}]")
        M = a.shape[0]
        if y is None:
            y = torch.empty((M, self.N), dtype=torch.bfloat16).pin_memory()
        if y.dtype != torch.bfloat16 or y.shape != (M, self.N) or not y.is_contiguous() or y.is_cuda:
            raise ValueError(f"y must be a contiguous host bf16 [{M}, {self.N}] tensor")
        _check(load_library().fp8_scaled_linear_host(self._h, M, a.data_ptr(), y.data_ptr(), _stream(self.device)))
        return y

    def forward_fp8(self, qa: torch.Tensor, sa: torch.Tensor, y: Optional[torch.Tensor] = None) -> torch.Tensor:
        if qa.dtype not in (torch.uint8, torch.float8_e4m3fn) or qa.dim() != 2 or not qa.is_contiguous():
            raise ValueError("qa must be contiguous E4M3FN codes [M, K]")
        if qa.shape[1] != self.K or sa.dtype != torch.float32 or sa.shape != (qa.shape[0],):
            raise ValueError("qa [M, K] and sa float32 [M] must match the layer")
        M = qa.shape[0]
        _same_device(qa, self.device, "qa")
        _same_device(sa, self.device, "sa")
        if not sa.is_contiguous():
            raise ValueError("sa must be contiguous")
        if y is None:
            y = torch.empty((M, self.N), dtype=torch.bfloat16, device=qa.device)
        _check_out(y, "y", _BF16_DTYPES, (M, self.N), qa.device)
        _check(load_library().fp8_scaled_linear(self._h, M, None, qa.data_ptr(), sa.data_ptr(), None, None,
                                                y.data_ptr(), _stream(qa.device)))
        return y


def scaled_linear_multi(layers: Sequence[FP8Linear], a: torch.Tensor,
                        ys: Optional[Sequence[torch.Tensor]] = None,
                        qa_scratch: Optional[torch.Tensor] = None,
                        sa_scratch: Optional[torch.Tensor] = None) -> List[torch.Tensor]:
    """Quantise ``a`` once and run every layer on it in one grouped launch
    ("从 BF16 到 FP8", section 三.4: Q / K / V share one activation quantisation)."""
    a = _bf16_matrix(a, "a")
    n = len(layers)
    M, K = a.shape
    if not a.is_contiguous():
        raise ValueError("a must be contiguous")
    for i, l in enumerate(layers):
        if l.K != K:
            raise ValueError(f"layers[{i}] has K = {l.K}, the activation {K}")
        _same_device(a, l.device, "a")
    if ys is None:
        ys = [torch.empty((M, l.N), dtype=torch.bfloat16, device=a.device) for l in layers]
    if qa_scratch is None:
        qa_scratch = torch.empty((M, K), dtype=torch.uint8, device=a.device)
    if sa_scratch is None:
        sa_scratch = torch.empty((M,), dtype=torch.float32, device=a.device)
    if len(ys) != n:
        raise ValueError("ys must hold one output per layer")
    for i, (y, l) in enumerate(zip(ys, layers)):
        _check_out(y, f"ys[{i}]", _BF16_DTYPES, (M, l.N), a.device)
    _check_out(qa_scratch, "qa_scratch", _CODE_DTYPES, (M, K), a.device)
    _check_out(sa_scratch, "sa_scratch", (torch.float32,), (M,), a.device)
    hs = (ctypes.c_void_p * n)(*[l.handle.value for l in layers])
    yp = (ctypes.c_void_p * n)(*[y.data_ptr() for y in ys])
    _check(load_library().fp8_scaled_linear_multi(hs, n, M, a.data_ptr(), qa_scratch.data_ptr(),
                                                  sa_scratch.data_ptr(), yp, _stream(a.device)))
    return list(ys)


def device_error(device: Optional[torch.device] = None) -> int:
    """Synchronise the current stream and read / clear the device error word (0 = OK, 5 = TIMEOUT)."""
    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    return int(load_library().fp8dit_device_error(_stream(dev)))


def selftest_expired_wait(limit_ns: int = 2_000_000, device: Optional[torch.device] = None) -> None:
    """Launch the bounded-wait self test (a wait that must expire)."""
    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    _check(load_library().fp8dit_selftest_expired_wait(limit_ns, _stream(dev)))


def selftest_quotient(device: Optional[torch.device] = None) -> Tuple[int, int]:
    """Run the exhaustive quotient self test; returns the FP8 code mismatch
    counts (E4M3FN, E5M2) against IEEE division (both must be 0)."""
    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    out = torch.zeros(2, dtype=torch.int64, device=dev)
    _check(load_library().fp8dit_selftest_quotient(out.data_ptr(), _stream(dev)))
    vals = out.cpu().tolist()
    return int(vals[0]), int(vals[1])
