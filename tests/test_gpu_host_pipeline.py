"""FP8 linear from host buffers (fp8_scaled_linear_host): chunked copy-in,
quantise + GEMM and copy-out on three streams.

Every chunk must give exactly what fp8_scaled_linear gives for the same rows
on the device (bit for bit), the rows must satisfy the oracle's tolerance,
and repeated and interleaved calls (slots reused across calls, two layers
alternating as in an FFN step) must each deliver their own result."""
import numpy as np
import pytest
import torch

import oracle
import synth
from conftest import bf16_tensor_to_f64, to_device_bf16

pytestmark = pytest.mark.gpu

fp8 = pytest.importorskip("dit_rowwise_amax_b200")


def host_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).pin_memory()


def make_layer(W, bias):
    qw, sw = fp8.quantize_weight_per_channel(to_device_bf16(W))
    layer = fp8.FP8Linear(qw, sw, None if bias is None else to_device_bf16(bias))
    torch.cuda.synchronize()
    return layer, qw.cpu().numpy(), sw.cpu().numpy()


def device_reference(layer, A, chunk):
    """fp8_scaled_linear on the device, one call per chunk of rows."""
    a = to_device_bf16(A)
    parts = [layer.forward(a[r0:r0 + chunk].contiguous()) for r0 in range(0, A.shape[0], chunk)]
    torch.cuda.synchronize()
    return torch.cat(parts).cpu()


def check_oracle(y, A, qw, sw, bias, rows):
    qa, sa = oracle.quantize_rows(np.ascontiguousarray(A[rows]), oracle.E4M3FN)
    ref = oracle.linear(qa, sa, qw, sw, bias)
    ok, worst = oracle.tolerance_ok(bf16_tensor_to_f64(y)[rows], ref)
    assert ok, f"tolerance exceeded: worst error / bound = {worst:.3f}"


@pytest.mark.parametrize("cfg", ["ffn_up", "ffn_down"])
def test_ffn_shapes_match_device_path(cfg):
    d = getattr(synth, cfg)()
    layer, qw, sw = make_layer(d["W"], d["bias"])
    layer.attach_host_pipeline(chunk_rows=512, slots=3)
    y = layer.forward_host(host_bf16(d["A"]))
    torch.cuda.synchronize()
    assert fp8.device_error() == 0
    assert torch.equal(y.view(torch.int16), device_reference(layer, d["A"], 512).view(torch.int16))
    M = d["A"].shape[0]
    rows = np.unique(np.concatenate([np.arange(16), np.arange(M - 16, M), np.arange(500, 530)]))
    check_oracle(y, d["A"], qw, sw, d["bias"], rows)


def test_ragged_rows_and_repeated_calls():
    M, N, K = 1000, 264, 2064
    W = synth.normal_bf16("gpu/host/W", (N, K), 0.02)
    bias = synth.normal_bf16("gpu/host/b", (N,), 0.1)
    layer, qw, sw = make_layer(W, bias)
    layer.attach_host_pipeline(chunk_rows=384, slots=2)  # chunks of 384, 384, 232; slots reused
    As = [synth.normal_bf16(f"gpu/host/A{i}", (M, K), 1.0, outlier_p=0.01, outlier_factor=20.0) for i in range(3)]
    # The host inputs must outlive the queued copies (the library reads them
    # asynchronously), so keep them referenced until the stream is synchronised.
    a_hosts = [host_bf16(A) for A in As]
    ys = [layer.forward_host(a) for a in a_hosts]  # three calls queued back to back
    torch.cuda.synchronize()
    for A, y in zip(As, ys):
        assert torch.equal(y.view(torch.int16), device_reference(layer, A, 384).view(torch.int16))
    check_oracle(ys[2], As[2], qw, sw, bias, np.arange(M))


def test_two_layers_interleaved():
    """Two layers alternating on one stream (an FFN step on host buffers): the
    second layer's copies overlap the first one's; every output must be its own."""
    up, down = synth.ffn_up(), synth.ffn_down()
    lu, _, _ = make_layer(up["W"], up["bias"])
    ld, _, _ = make_layer(down["W"], down["bias"])
    lu.attach_host_pipeline(chunk_rows=1024, slots=2)
    ld.attach_host_pipeline(chunk_rows=1024, slots=2)
    au, ad = host_bf16(up["A"]), host_bf16(down["A"])
    outs = []
    for _ in range(3):
        outs.append((lu.forward_host(au), ld.forward_host(ad)))
    torch.cuda.synchronize()
    ref_u = device_reference(lu, up["A"], 1024)
    ref_d = device_reference(ld, down["A"], 1024)
    for yu, yd in outs:
        assert torch.equal(yu.view(torch.int16), ref_u.view(torch.int16))
        assert torch.equal(yd.view(torch.int16), ref_d.view(torch.int16))


def test_argument_errors():
    L = fp8.load_library()
    W = synth.normal_bf16("gpu/host/err/W", (64, 128), 0.02)
    layer, _, _ = make_layer(W, None)
    a = host_bf16(synth.normal_bf16("gpu/host/err/A", (16, 128), 1.0))
    y = torch.empty((16, 64), dtype=torch.bfloat16).pin_memory()
    s = fp8._stream(torch.device("cuda"))
    h = layer.handle
    assert L.fp8_scaled_linear_host(h, 16, a.data_ptr(), y.data_ptr(), s) == 1  # nothing attached
    assert L.fp8_linear_host_workspace_size(h, 0, 2) == 0
    assert L.fp8_linear_host_workspace_size(h, 64, 1) == 0
    need = int(L.fp8_linear_host_workspace_size(h, 64, 2))
    ws = torch.empty((need + 512,), dtype=torch.uint8, device="cuda")
    assert L.fp8_linear_set_host_pipeline(h, ws.data_ptr() + 16, need, 64, 2) == 1  # misaligned
    assert L.fp8_linear_set_host_pipeline(h, ws.data_ptr(), need - 1, 64, 2) == 1   # too small
    assert L.fp8_linear_set_host_pipeline(h, ws.data_ptr(), need, 64, 9) == 1       # slots
    assert L.fp8_linear_set_host_pipeline(h, ws.data_ptr(), need, 64, 2) == 0
    assert L.fp8_scaled_linear_host(h, 16, None, y.data_ptr(), s) == 1
    assert L.fp8_scaled_linear_host(h, -1, a.data_ptr(), y.data_ptr(), s) == 1
    assert L.fp8_scaled_linear_host(h, 0, None, None, s) == 0
    assert L.fp8_scaled_linear_host(h, 16, a.data_ptr(), y.data_ptr(), s) == 0
    torch.cuda.synchronize()
    assert L.fp8_linear_set_host_pipeline(h, None, 0, 0, 0) == 0  # detach
    assert L.fp8_scaled_linear_host(h, 16, a.data_ptr(), y.data_ptr(), s) == 1
    assert fp8.device_error() == 0


def test_reattach_while_work_in_flight():
    """Re-attaching a pipeline to the same workspace while a call is still
    queued waits for that call's work, so neither result is corrupted."""
    M, N, K = 2048, 512, 1024
    W = synth.normal_bf16("gpu/host/re/W", (N, K), 0.02)
    layer, _, _ = make_layer(W, None)
    ws = layer.attach_host_pipeline(chunk_rows=256, slots=2)
    L = fp8.load_library()
    A0 = synth.normal_bf16("gpu/host/re/A0", (M, K), 1.0)
    A1 = synth.normal_bf16("gpu/host/re/A1", (M, K), 1.0)
    a0, a1 = host_bf16(A0), host_bf16(A1)
    y0 = layer.forward_host(a0)                 # queued, not synchronised
    assert L.fp8_linear_set_host_pipeline(layer.handle, ws.data_ptr(), ws.numel(), 256, 2) == 0
    y1 = layer.forward_host(a1)
    torch.cuda.synchronize()
    assert torch.equal(y0.view(torch.int16), device_reference(layer, A0, 256).view(torch.int16))
    assert torch.equal(y1.view(torch.int16), device_reference(layer, A1, 256).view(torch.int16))
