"""The FP8 linear from a bf16 activation in one launch (fp8_scaled_linear_fused)
on the GPU vs the CPU oracle.

The launch's CTAs first quantise A per token (each element once) into the
caller's scratch, then run the GEMM. The codes and scales it writes must equal
the oracle's bit for bit; the output is compared with the oracle's exact
product of the oracle's own codes (|gpu - ref| <= 1e-2 |ref| + 1e-3 rms(ref))
and, where both run 256 x 256 pair tiles, with the two-launch
fp8_scaled_linear bit for bit. Every launch must leave the workspace's
counters at zero, so repeated calls and CUDA-graph replays need no reset."""

import numpy as np
import pytest
import torch

import oracle
import synth
from conftest import bf16_tensor_to_f64, to_device_bf16

pytestmark = pytest.mark.gpu

fp8 = pytest.importorskip("dit_rowwise_amax_b200")


def make_layer(W, bias):
    qw, sw = fp8.quantize_weight_per_channel(to_device_bf16(W))
    layer = fp8.FP8Linear(qw, sw, None if bias is None else to_device_bf16(bias))
    torch.cuda.synchronize()
    return layer, qw.cpu().numpy(), sw.cpu().numpy()


def run_fused(layer, A):
    M, K = A.shape
    qa = torch.full((M, K), 0xCD, dtype=torch.uint8, device="cuda")
    sa = torch.full((M,), -1.0, dtype=torch.float32, device="cuda")
    y = layer.forward_fused(to_device_bf16(A), qa_scratch=qa, sa_scratch=sa)
    torch.cuda.synchronize()
    assert fp8.device_error() == 0
    qo, so = oracle.quantize_rows(A, oracle.E4M3FN)
    assert np.array_equal(sa.cpu().numpy().view(np.uint32), so.view(np.uint32)), "per-token scales differ"
    assert np.array_equal(qa.cpu().numpy(), qo), "codes differ"
    return y, qo, so


def check_rows(y, qa, sa, qw, sw, bias, rows):
    ref = oracle.linear(np.ascontiguousarray(qa[rows]), sa[rows], qw, sw, bias)
    ok, worst = oracle.tolerance_ok(bf16_tensor_to_f64(y)[rows], ref)
    assert ok, f"tolerance exceeded: worst error / bound = {worst:.3f}"


def counters_zero(layer):
    flag_bytes = layer.workspace_flag_bytes()  # the flags and counters at the start of the workspace
    assert 0 < flag_bytes < layer.workspace.numel()
    return int(torch.count_nonzero(layer.workspace[:flag_bytes])) == 0


@pytest.mark.parametrize("cfg", ["ffn_up", "ffn_down"])
def test_ffn_full_size_matches_unfused_bitwise(cfg):
    d = getattr(synth, cfg)()
    layer, qw, sw = make_layer(d["W"], d["bias"])
    M = d["A"].shape[0]
    y, qa, sa = run_fused(layer, d["A"])
    layer.detach_workspace()
    assert layer.plan(M)[:2] == (256, 256)
    y_ref = layer.forward(to_device_bf16(d["A"]))
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16)), "fused and unfused outputs differ"
    check_rows(y, qa, sa, qw, sw, d["bias"], np.arange(M))


def test_tiny_config_full():
    d = synth.tiny()
    layer, qw, sw = make_layer(d["W"], d["bias"])
    y, qa, sa = run_fused(layer, d["A"])
    check_rows(y, qa, sa, qw, sw, d["bias"], np.arange(64))
    assert counters_zero(layer)


@pytest.mark.parametrize("M", [1, 26, 129, 257, 300])
@pytest.mark.parametrize("N,K", [(8, 16), (136, 48), (520, 2064), (2048, 2048), (264, 8192)])
def test_ragged_shapes(M, N, K):
    A = synth.normal_bf16(f"gpu/fused/A/{M}x{K}", (M, K), 1.0, outlier_p=0.01, outlier_factor=20.0)
    W = synth.normal_bf16(f"gpu/fused/W/{N}x{K}", (N, K), 0.02)
    bias = synth.normal_bf16(f"gpu/fused/b/{N}", (N,), 0.1)
    layer, qw, sw = make_layer(W, bias)
    y, qa, sa = run_fused(layer, A)
    check_rows(y, qa, sa, qw, sw, bias, np.arange(M))
    assert counters_zero(layer)


def test_special_rows():
    """All-zero and all -0 rows (S = 1), a constant row, rows whose amax is
    below 2^-64 (exact-division quotient), bf16 subnormals, in a ragged
    300 x 2064 activation spanning two pair tiles."""
    M, N, K = 300, 264, 2064
    A = synth.normal_bf16("gpu/fused/special/A", (M, K), 1.0, outlier_p=0.01, outlier_factor=30.0).copy()
    A[0] = 0x0000                       # +0
    A[1] = 0x8000                       # -0
    A[2] = 0x3F00                       # 0.5 everywhere
    tiny = synth.normal_bf16("gpu/fused/special/tiny", (4, K), 1.0)
    f = synth.bf16_to_f32(tiny) * np.float32(2.0 ** -70)
    A[3:7] = (f.view(np.uint32) >> 16).astype(np.uint16)  # amax ~ 2^-68 (truncated to bf16)
    A[7] = np.where(np.arange(K) % 2 == 0, 0x0001, 0x8003).astype(np.uint16)  # bf16 subnormals only
    A[257] = 0x0000                     # a zero row in the second pair tile
    W = synth.normal_bf16("gpu/fused/special/W", (N, K), 0.02)
    bias = synth.normal_bf16("gpu/fused/special/b", (N,), 0.1)
    layer, qw, sw = make_layer(W, bias)
    y, qa, sa = run_fused(layer, A)
    assert sa[0] == 1.0 and sa[1] == 1.0 and sa[257] == 1.0
    check_rows(y, qa, sa, qw, sw, bias, np.arange(M))


def test_repeated_calls_and_graph_replays():
    """Stream-ordered calls and replays of a captured graph, with new inputs
    between replays: every result equals the first call's for the same input,
    and the counters are back at zero after each."""
    M, N, K = 1000, 2048, 2048
    W = synth.normal_bf16("gpu/fused/graph/W", (N, K), 0.02)
    layer, _, _ = make_layer(W, synth.normal_bf16("gpu/fused/graph/b", (N,), 0.1))
    As = [to_device_bf16(synth.normal_bf16(f"gpu/fused/graph/A{i}", (M, K), 1.0)) for i in range(3)]
    refs = [layer.forward_fused(a) for a in As]
    torch.cuda.synchronize()
    assert counters_zero(layer)
    for _ in range(2):
        for a, r in zip(As, refs):
            assert torch.equal(layer.forward_fused(a).view(torch.int16), r.view(torch.int16))
    a_in = As[0].clone()
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    qa = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    sa = torch.empty((M,), dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        layer.forward_fused(a_in, y=y, qa_scratch=qa, sa_scratch=sa)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        layer.forward_fused(a_in, y=y, qa_scratch=qa, sa_scratch=sa)
    for i in (1, 2, 0):
        a_in.copy_(As[i])
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), refs[i].view(torch.int16)), f"replay with input {i}"
    del g
    assert fp8.device_error() == 0
    assert counters_zero(layer)


def test_argument_errors_launch_nothing():
    L = fp8.load_library()
    W = synth.normal_bf16("gpu/fused/err/W", (64, 128), 0.02)
    layer, _, _ = make_layer(W, None)
    a = to_device_bf16(synth.normal_bf16("gpu/fused/err/A", (16, 128), 1.0))
    y = torch.full((16, 64), 3.0, dtype=torch.bfloat16, device="cuda")
    qa = torch.empty((16, 128), dtype=torch.uint8, device="cuda")
    sa = torch.empty((16,), dtype=torch.float32, device="cuda")
    s = fp8._stream(a.device)
    # No workspace attached yet: refused.
    assert L.fp8_scaled_linear_fused(layer.handle, 16, a.data_ptr(), qa.data_ptr(), sa.data_ptr(), y.data_ptr(), s) == 1
    layer.attach_workspace()
    assert L.fp8_scaled_linear_fused(layer.handle, 16, a.data_ptr(), None, sa.data_ptr(), y.data_ptr(), s) == 1
    assert L.fp8_scaled_linear_fused(layer.handle, 16, a.data_ptr(), qa.data_ptr(), sa.data_ptr() + 2, y.data_ptr(), s) == 1
    assert L.fp8_scaled_linear_fused(layer.handle, 16, a.data_ptr() + 8, qa.data_ptr(), sa.data_ptr(), y.data_ptr(), s) == 1
    assert L.fp8_scaled_linear_fused(layer.handle, 16, a.data_ptr(), qa.data_ptr() + 8, sa.data_ptr(), y.data_ptr(), s) == 1
    assert L.fp8_scaled_linear_fused(layer.handle, -1, a.data_ptr(), qa.data_ptr(), sa.data_ptr(), y.data_ptr(), s) == 1
    assert L.fp8_scaled_linear_fused(layer.handle, 0, None, None, None, None, s) == 0
    assert L.fp8_scaled_linear_fused(None, 16, a.data_ptr(), qa.data_ptr(), sa.data_ptr(), y.data_ptr(), s) == 1
    torch.cuda.synchronize()
    assert bool(torch.all(y == 3.0)), "a refused call wrote its output"
    assert fp8.device_error() == 0


def test_long_rows_refused():
    """Rows longer than 8192 elements do not fit the launch's staging: refused
    with UNSUPPORTED_SHAPE, nothing written."""
    L = fp8.load_library()
    M, N, K = 8, 64, 8208
    layer, _, _ = make_layer(synth.normal_bf16("gpu/fused/long/W", (N, K), 0.02), None)
    layer.attach_workspace()
    a = to_device_bf16(synth.normal_bf16("gpu/fused/long/A", (M, K), 1.0))
    y = torch.full((M, N), 3.0, dtype=torch.bfloat16, device="cuda")
    qa = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    sa = torch.empty((M,), dtype=torch.float32, device="cuda")
    st = L.fp8_scaled_linear_fused(layer.handle, M, a.data_ptr(), qa.data_ptr(), sa.data_ptr(), y.data_ptr(),
                                   fp8._stream(a.device))
    assert st == 2
    torch.cuda.synchronize()
    assert bool(torch.all(y == 3.0))
