"""Stream-K schedule of the FP8 GEMM (a layer with an attached workspace whose
256 x 256 tiles would keep the CTA pairs busy for less than 3/4 of a
tile-per-pair schedule): parity with the oracle, the same result on every run,
and a different summation split from the plain schedule (which shows the split
actually ran). Shapes outside that rule keep the plain schedule bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import synth
from conftest import bf16_tensor_to_f64, to_device_bf16

pytestmark = pytest.mark.gpu

fp8 = pytest.importorskip("dit_rowwise_amax_b200")


def layer_and_codes(W, bias):
    qw, sw = fp8.quantize_weight_per_channel(to_device_bf16(W))
    layer = fp8.FP8Linear(qw, sw, to_device_bf16(bias))
    torch.cuda.synchronize()
    return layer, qw.cpu().numpy(), sw.cpu().numpy()


def check_rows(y, qa, sa, qw, sw, bias, rows):
    ref = oracle.linear(np.ascontiguousarray(qa[rows]), sa[rows], qw, sw, bias)
    ok, worst = oracle.tolerance_ok(bf16_tensor_to_f64(y)[rows], ref)
    assert ok, f"tolerance exceeded: worst error / bound = {worst:.3f}"


# 152 tiles (19 x 8), 9 k-blocks, ragged M; 165 tiles (11 x 15) with ragged M,
# N and K; 152 tiles at the FFN-down width and depth.
@pytest.mark.parametrize("M,N,K", [(4800, 2048, 1040), (2600, 3776, 4160), (4864, 2048, 8192)])
def test_stream_k_parity_and_determinism(M, N, K):
    A = synth.normal_bf16(f"gpu/sk/A/{M}x{K}", (M, K), 1.0, outlier_p=0.01, outlier_factor=20.0)
    W = synth.ffn_down()["W"] if (N, K) == (2048, 8192) else synth.normal_bf16(f"gpu/sk/W/{N}x{K}", (N, K), 0.02)
    bias = synth.normal_bf16(f"gpu/sk/b/{N}", (N,), 0.1)
    layer, qw, sw = layer_and_codes(W, bias)
    qa_d, sa_d = fp8.quantize_rowwise(to_device_bf16(A))
    y_plain = layer.forward_fp8(qa_d, sa_d)
    layer.attach_workspace()
    y1 = layer.forward_fp8(qa_d, sa_d)
    y2 = layer.forward_fp8(qa_d, sa_d)
    torch.cuda.synchronize()
    assert fp8.device_error() == 0
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16)), "stream-K result changed between runs"
    assert not torch.equal(y1.view(torch.int16), y_plain.view(torch.int16)), "no tile was split"
    qa, sa = qa_d.cpu().numpy(), sa_d.cpu().numpy()
    check_rows(y1, qa, sa, qw, sw, bias, np.arange(M))  # every output
    layer.detach_workspace()
    y3 = layer.forward_fp8(qa_d, sa_d)
    torch.cuda.synchronize()
    assert torch.equal(y3.view(torch.int16), y_plain.view(torch.int16))


def test_workspace_argument_checks():
    L = fp8.load_library()
    W = synth.normal_bf16("gpu/sk/w2", (256, 256), 0.02)
    layer, _, _ = layer_and_codes(W, synth.normal_bf16("gpu/sk/b2", (256,), 0.1))
    need = int(L.fp8_linear_workspace_size(layer.handle))
    assert need > 0
    ws = torch.empty(need + 512, dtype=torch.uint8, device="cuda")
    assert L.fp8_linear_set_workspace(layer.handle, ws.data_ptr() + 16, need) == 1  # misaligned
    assert L.fp8_linear_set_workspace(layer.handle, ws.data_ptr(), need - 1) == 1   # too small
    assert L.fp8_linear_set_workspace(layer.handle, ws.data_ptr(), need) == 0
    assert L.fp8_linear_set_workspace(layer.handle, None, 0) == 0


def test_ffn_shapes_keep_plain_schedule():
    """FFN-down (128 tiles: 86% of two waves busy) is faster data-parallel, so
    an attached workspace leaves its result bit-identical."""
    d = synth.ffn_down()
    layer, _, _ = layer_and_codes(d["W"], d["bias"])
    qa_d, sa_d = fp8.quantize_rowwise(to_device_bf16(d["A"]))
    y_plain = layer.forward_fp8(qa_d, sa_d)
    layer.attach_workspace()
    y_ws = layer.forward_fp8(qa_d, sa_d)
    torch.cuda.synchronize()
    assert torch.equal(y_ws.view(torch.int16), y_plain.view(torch.int16))


def test_stream_k_cuda_graph_replays():
    """Stream-K launches replayed from a captured CUDA graph: every launch
    leaves the workspace flags cleared, so each replay (with new inputs copied
    into the captured buffers) equals the eager result for those inputs."""
    M, N, K = 4800, 2048, 1040  # 152 pair tiles: the split schedule
    W = synth.normal_bf16(f"gpu/sk/W/{N}x{K}", (N, K), 0.02)
    layer, _, _ = layer_and_codes(W, synth.normal_bf16(f"gpu/sk/b/{N}", (N,), 0.1))
    layer.attach_workspace()
    inputs = [fp8.quantize_rowwise(to_device_bf16(synth.normal_bf16(f"gpu/sk/graph/A{i}", (M, K), 1.0)))
              for i in range(3)]
    eager = [layer.forward_fp8(qa, sa) for qa, sa in inputs]
    torch.cuda.synchronize()
    qa_buf, sa_buf = inputs[0][0].clone(), inputs[0][1].clone()
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        layer.forward_fp8(qa_buf, sa_buf, y=y)  # warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        layer.forward_fp8(qa_buf, sa_buf, y=y)
    for rep in range(2):
        for (qa, sa), ref in zip(inputs, eager):
            qa_buf.copy_(qa)
            sa_buf.copy_(sa)
            g.replay()
            torch.cuda.synchronize()
            assert fp8.device_error() == 0
            assert torch.equal(y.view(torch.int16), ref.view(torch.int16)), f"replay {rep} differs"


def test_stream_k_concurrent_launches_leave_marks_cleared():
    """Stream-K launches of two layers (each with its own workspace) on two
    streams at once, beside a pair-tile GEMM on a third: a split tile is
    finished by whichever of its two units gets there second, so nothing
    waits on a unit that has not started. Every output equals the same call
    run alone, bit for bit; no device error; every mark is back at zero."""
    M, N, K = 4864, 2048, 8192
    d = synth.ffn_down()
    layers, acts, refs = [], [], []
    for i in range(2):
        layer, _, _ = layer_and_codes(d["W"], synth.normal_bf16(f"gpu/sk/conc/b{i}", (N,), 0.1))
        layer.attach_workspace()
        qa, sa = fp8.quantize_rowwise(to_device_bf16(synth.normal_bf16(f"gpu/sk/conc/A{i}", (M, K), 1.0)))
        layers.append(layer)
        acts.append((qa, sa))
        refs.append(layer.forward_fp8(qa, sa))
    u = synth.ffn_up()
    big = fp8.FP8Linear.from_weight(to_device_bf16(u["W"]), to_device_bf16(u["bias"]))
    big_q = fp8.quantize_rowwise(to_device_bf16(u["A"]))
    torch.cuda.synchronize()
    assert fp8.device_error() == 0
    streams = [torch.cuda.Stream() for _ in range(3)]
    outs = [[torch.empty((M, N), dtype=torch.bfloat16, device="cuda") for _ in range(6)] for _ in range(2)]
    for it in range(6):
        with torch.cuda.stream(streams[2]):
            big.forward_fp8(*big_q)
        for i in range(2):
            with torch.cuda.stream(streams[i]):
                layers[i].forward_fp8(*acts[i], y=outs[i][it])
    torch.cuda.synchronize()
    assert fp8.device_error() == 0
    for i in range(2):
        for it in range(6):
            assert torch.equal(outs[i][it].view(torch.int16), refs[i].view(torch.int16)), (i, it)
        nb = layers[i].workspace_flag_bytes()
        assert int(torch.count_nonzero(layers[i].workspace[:nb])) == 0
