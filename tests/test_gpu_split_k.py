"""Split-K schedule of the FP8 GEMM for few output tiles and a long K (small
M, e.g. text tokens through an FFN-down weight). With a workspace attached,
128 x 128 tiles filling at most half of the SMs and at least 48 k-blocks, each
tile is cut into pieces along K on separate CTAs; every piece stores its fp32
partial and arrives on the tile's counter, and the piece that arrives last adds
all of them in piece order and writes the tile. Checked: the plan reports the
split, every output against the oracle, the same bits on every run, no write
outside y, graph replays, one workspace shared with stream-K, concurrent
launches on several streams, counters left cleared, and the plain schedule
after detach and for a short K."""
import numpy as np
import pytest
import torch

import oracle
import synth
from conftest import bf16_tensor_to_f64, canary_buffer, check_canary, to_device_bf16

pytestmark = pytest.mark.gpu

fp8 = pytest.importorskip("dit_rowwise_amax_b200")


def layer_and_codes(W, bias):
    qw, sw = fp8.quantize_weight_per_channel(to_device_bf16(W))
    layer = fp8.FP8Linear(qw, sw, to_device_bf16(bias))
    torch.cuda.synchronize()
    return layer, qw.cpu().numpy(), sw.cpu().numpy()


def tiles128(M, N, n=1):
    return -(-M // 128) * -(-N // 128) * n


def check_all(y, qa, sa, qw, sw, bias):
    ref = oracle.linear(qa, sa, qw, sw, bias)
    ok, worst = oracle.tolerance_ok(bf16_tensor_to_f64(y), ref)
    assert ok, f"tolerance exceeded: worst error / bound = {worst:.3f}"


# One token; the encoder_hidden_states length at FFN-down depth; ragged N (a
# last tile 8 columns wide) with ragged K (65 k-blocks, the last one 16
# elements); a full 128-row tile; two row tiles at the shortest split K; 48
# tiles (3 pieces each).
@pytest.mark.parametrize("M,N,K", [(1, 2048, 8192), (26, 2048, 8192), (100, 264, 8208), (128, 2048, 8192),
                                   (200, 1024, 6144), (26, 6144, 8192)])
def test_split_k_parity_and_determinism(M, N, K):
    A = synth.normal_bf16(f"gpu/split/A/{M}x{K}", (M, K), 1.0, outlier_p=0.01, outlier_factor=20.0)
    W = synth.normal_bf16(f"gpu/split/W/{N}x{K}", (N, K), 0.02)
    bias = synth.normal_bf16(f"gpu/split/b/{N}", (N,), 0.1)
    layer, qw, sw = layer_and_codes(W, bias)
    qa_d, sa_d = fp8.quantize_rowwise(to_device_bf16(A))
    plain_plan = layer.plan(M)
    y_plain = layer.forward_fp8(qa_d, sa_d)
    layer.attach_workspace()
    bm, bn, ctas = layer.plan(M)
    assert (bm, bn) == (128, 128) and ctas > tiles128(M, N) and ctas <= torch.cuda.get_device_properties(0).multi_processor_count
    nbytes = M * N * 2
    buf, view = canary_buffer(nbytes)
    y1 = view.view(torch.bfloat16).view(M, N)
    layer.forward_fp8(qa_d, sa_d, y=y1)
    y2 = layer.forward_fp8(qa_d, sa_d)
    torch.cuda.synchronize()
    assert fp8.device_error() == 0
    check_canary(buf, nbytes)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16)), "split-K result changed between runs"
    check_all(y1, qa_d.cpu().numpy(), sa_d.cpu().numpy(), qw, sw, bias)
    layer.detach_workspace()
    assert layer.plan(M) == plain_plan
    y3 = layer.forward_fp8(qa_d, sa_d)
    torch.cuda.synchronize()
    assert torch.equal(y3.view(torch.int16), y_plain.view(torch.int16))


def test_split_k_from_bf16_and_multi():
    """Three layers sharing K = 8192 in one grouped launch at M = 26 with the
    first layer's workspace (48 tiles, 3 pieces each), and each layer alone
    from the bf16 activation (16 tiles, 8 pieces each): every output against
    the oracle."""
    M, N, K = 26, 2048, 8192
    A = synth.normal_bf16("gpu/split/multi/A", (M, K), 1.0, outlier_p=0.01, outlier_factor=20.0)
    layers, codes = [], []
    for p in "qkv":
        W = synth.normal_bf16(f"gpu/split/multi/W{p}", (N, K), 0.015)
        bias = synth.normal_bf16(f"gpu/split/multi/b{p}", (N,), 0.1)
        layer, qw, sw = layer_and_codes(W, bias)
        layers.append(layer)
        codes.append((qw, sw, bias))
    ws = layers[0].attach_workspace()
    assert layers[0].plan(M, 3)[2] == 48 * 3
    qa, sa = oracle.quantize_rows(A, oracle.E4M3FN)
    ys = fp8.scaled_linear_multi(layers, to_device_bf16(A))
    torch.cuda.synchronize()
    assert fp8.device_error() == 0
    for y, (qw, sw, bias) in zip(ys, codes):
        check_all(y, qa, sa, qw, sw, bias)
    for layer in layers[1:]:
        layer.attach_workspace(ws)
    singles = [layer.forward(to_device_bf16(A)) for layer in layers]
    torch.cuda.synchronize()
    assert fp8.device_error() == 0
    for y, (qw, sw, bias) in zip(singles, codes):
        check_all(y, qa, sa, qw, sw, bias)


def test_split_k_cuda_graph_replays():
    """Split-K launches replayed from a captured CUDA graph: the CTA that draws
    a tile's last ticket resets the counter, so each replay (new inputs copied
    into the captured buffers) equals the eager result."""
    M, N, K = 26, 2048, 8192
    W = synth.normal_bf16(f"gpu/split/W/{N}x{K}", (N, K), 0.02)
    layer, _, _ = layer_and_codes(W, synth.normal_bf16(f"gpu/split/b/{N}", (N,), 0.1))
    layer.attach_workspace()
    assert layer.plan(M)[2] > 16
    inputs = [fp8.quantize_rowwise(to_device_bf16(synth.normal_bf16(f"gpu/split/graph/A{i}", (M, K), 1.0)))
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
        for _ in range(3):  # back-to-back launches sharing the workspace
            layer.forward_fp8(qa_buf, sa_buf, y=y)
    for rep in range(2):
        for (qa, sa), ref in zip(inputs, eager):
            qa_buf.copy_(qa)
            sa_buf.copy_(sa)
            g.replay()
            torch.cuda.synchronize()
            assert fp8.device_error() == 0
            assert torch.equal(y.view(torch.int16), ref.view(torch.int16)), f"replay {rep} differs"


@pytest.mark.parametrize("M,N,K", [(200, 8192, 8192), (26, 2048, 2048)])
def test_split_k_leaves_other_plans_alone(M, N, K):
    """Enough tiles to fill the SMs (2 x 64 = 128 tiles of 128 x 128 > SMs / 2),
    or too short a K (16 k-blocks; 128 x 64 tiles): an attached workspace
    changes neither the plan nor the bits of a single-CTA launch."""
    W = synth.normal_bf16(f"gpu/split/W/{N}x{K}", (N, K), 0.02)
    layer, _, _ = layer_and_codes(W, synth.normal_bf16(f"gpu/split/b/{N}", (N,), 0.1))
    qa_d, sa_d = fp8.quantize_rowwise(to_device_bf16(synth.normal_bf16("gpu/split/large/A", (M, K), 1.0)))
    plan = layer.plan(M)
    assert plan[:2] == ((128, 128) if N * M > 2048 * 128 else (128, 64))
    y_plain = layer.forward_fp8(qa_d, sa_d)
    layer.attach_workspace()
    assert layer.plan(M) == plan
    y_ws = layer.forward_fp8(qa_d, sa_d)
    torch.cuda.synchronize()
    assert torch.equal(y_ws.view(torch.int16), y_plain.view(torch.int16))


def test_one_workspace_for_mixed_plans():
    """One workspace shared, in stream order, by split-K launches of 16 and of 48
    tiles (FP8 and weight-only) and by stream-K launches (152 pair tiles), in an order where each
    plan follows the others: every result equals the same layer's result on a
    workspace of its own, bit for bit, and no bounded wait expires. (The
    split-K counters and the stream-K flags occupy separate, fixed regions.)"""
    K = 8192
    W16 = synth.normal_bf16("gpu/split/mixed/W16", (2048, K), 0.02)
    W48 = synth.normal_bf16("gpu/split/mixed/W48", (6144, K), 0.02)
    Wsk = synth.normal_bf16("gpu/split/mixed/Wsk", (2048, 1040), 0.02)
    l16, _, _ = layer_and_codes(W16, synth.normal_bf16("gpu/split/mixed/b16", (2048,), 0.1))
    l48, _, _ = layer_and_codes(W48, synth.normal_bf16("gpu/split/mixed/b48", (6144,), 0.1))
    lsk, _, _ = layer_and_codes(Wsk, synth.normal_bf16("gpu/split/mixed/bsk", (2048,), 0.1))
    a_small = fp8.quantize_rowwise(to_device_bf16(synth.normal_bf16("gpu/split/mixed/A", (26, K), 1.0)))
    a_sk = fp8.quantize_rowwise(to_device_bf16(synth.normal_bf16("gpu/split/mixed/Ask", (4800, 1040), 1.0)))
    a_bf16 = to_device_bf16(synth.normal_bf16("gpu/split/mixed/Awo", (26, K), 1.0))
    runs = {"16": (l16, a_small), "48": (l48, a_small), "sk": (lsk, a_sk), "wo": (l48, a_bf16)}

    def call(name):
        layer, arg = runs[name]
        return layer.forward_weight_only(arg) if name == "wo" else layer.forward_fp8(*arg)

    ref = {}
    for name, (layer, _) in runs.items():
        torch.cuda.synchronize()  # attach only while no call of the layer is in flight
        layer.attach_workspace()  # a private workspace
        ref[name] = call(name)
    torch.cuda.synchronize()
    assert fp8.device_error() == 0
    assert l16.plan(26)[2] > 16 and l48.plan(26)[2] > 48  # both split
    torch.cuda.synchronize()
    ws = l16.attach_workspace()
    l48.attach_workspace(ws)
    lsk.attach_workspace(ws)
    for name in ["16", "48", "wo", "16", "sk", "48", "wo", "sk", "16", "48"]:
        y = call(name)
        torch.cuda.synchronize()
        assert fp8.device_error() == 0, f"a bounded wait expired in the {name} launch"
        assert torch.equal(y.view(torch.int16), ref[name].view(torch.int16)), name


# FP8 weight-only linear (bf16 activation, E4M3 weight decoded in shared
# memory): the same split with 64-element k-blocks, from 32 k-blocks on (64
# above 64 rows). Ragged N and K at M = 60: 33 k-blocks, the last 16 elements.
@pytest.mark.parametrize("M,N,K", [(1, 2048, 2048), (26, 2048, 8192), (60, 264, 2064), (128, 2048, 4096)])
def test_weight_only_split_k(M, N, K):
    A = synth.normal_bf16(f"gpu/split/wo/A/{M}x{K}", (M, K), 1.0, outlier_p=0.01, outlier_factor=20.0)
    W = synth.normal_bf16(f"gpu/split/wo/W/{N}x{K}", (N, K), 0.02)
    bias = synth.normal_bf16(f"gpu/split/wo/b/{N}", (N,), 0.1)
    layer, qw, sw = layer_and_codes(W, bias)
    a = to_device_bf16(A)
    y_plain = layer.forward_weight_only(a)
    layer.attach_workspace()
    nbytes = M * N * 2
    buf, view = canary_buffer(nbytes)
    y1 = view.view(torch.bfloat16).view(M, N)
    layer.forward_weight_only(a, y=y1)
    y2 = layer.forward_weight_only(a)
    torch.cuda.synchronize()
    assert fp8.device_error() == 0
    check_canary(buf, nbytes)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16)), "split-K result changed between runs"
    ref = oracle.linear_weight_only(A, qw, sw, bias)
    ok, worst = oracle.tolerance_ok(bf16_tensor_to_f64(y1), ref)
    assert ok, f"tolerance exceeded: worst error / bound = {worst:.3f}"
    if K >= 8192:  # tens of thousands of outputs: a different summation split shows in some bits
        assert not torch.equal(y1.view(torch.int16), y_plain.view(torch.int16)), "no tile was split"
    layer.detach_workspace()
    y3 = layer.forward_weight_only(a)
    torch.cuda.synchronize()
    assert torch.equal(y3.view(torch.int16), y_plain.view(torch.int16))


def test_split_k_concurrent_launches_on_two_streams():
    """Split-K launches of two layers (each with its own workspace) issued on
    two streams so that they share the GPU, alongside a pair-tile GEMM on a
    third stream. No piece waits for another (the last piece to arrive reduces
    its tile), so nothing depends on all of a launch's CTAs being resident at
    once: every launch completes, no device error is raised, and every output
    equals the same call run alone, bit for bit."""
    M, N, K = 26, 2048, 8192
    layers, acts, refs = [], [], []
    for i in range(2):
        W = synth.normal_bf16(f"gpu/split/conc/W{i}", (N, K), 0.02)
        layer, _, _ = layer_and_codes(W, synth.normal_bf16(f"gpu/split/conc/b{i}", (N,), 0.1))
        layer.attach_workspace()
        qa, sa = fp8.quantize_rowwise(to_device_bf16(synth.normal_bf16(f"gpu/split/conc/A{i}", (M, K), 1.0)))
        layers.append(layer)
        acts.append((qa, sa))
        refs.append(layer.forward_fp8(qa, sa))
    d = synth.ffn_up()
    big = fp8.FP8Linear.from_weight(to_device_bf16(d["W"]), to_device_bf16(d["bias"]))
    big_q = fp8.quantize_rowwise(to_device_bf16(d["A"]))
    torch.cuda.synchronize()
    assert fp8.device_error() == 0
    streams = [torch.cuda.Stream() for _ in range(3)]
    outs = [[torch.empty((M, N), dtype=torch.bfloat16, device="cuda") for _ in range(20)] for _ in range(2)]
    for it in range(20):
        with torch.cuda.stream(streams[2]):
            big.forward_fp8(*big_q)
        for i in range(2):
            with torch.cuda.stream(streams[i]):
                layers[i].forward_fp8(*acts[i], y=outs[i][it])
    torch.cuda.synchronize()
    assert fp8.device_error() == 0
    for i in range(2):
        for it in range(20):
            assert torch.equal(outs[i][it].view(torch.int16), refs[i].view(torch.int16)), (i, it)


def test_split_k_leaves_counters_cleared():
    """Every launch returns the workspace's flag area (stream-K flags and the
    split-K arrival counters) to zero, so stream-ordered launches need no host
    reset: after split-K launches of several shapes the area reads all zero."""
    K = 8192
    W = synth.normal_bf16(f"gpu/split/W/2048x{K}", (2048, K), 0.02)
    layer, _, _ = layer_and_codes(W, synth.normal_bf16("gpu/split/b/2048", (2048,), 0.1))
    ws = layer.attach_workspace()
    for M in (1, 26, 128, 300):
        qa, sa = fp8.quantize_rowwise(to_device_bf16(synth.normal_bf16(f"gpu/split/clr/A{M}", (M, K), 1.0)))
        layer.forward_fp8(qa, sa)
        layer.forward_weight_only(to_device_bf16(synth.normal_bf16(f"gpu/split/clr/A16{M}", (M, K), 1.0)))
    torch.cuda.synchronize()
    assert fp8.device_error() == 0
    flag_bytes = layer.workspace_flag_bytes()  # the flags and counters at the start of the workspace
    assert 0 < flag_bytes < ws.numel()
    assert int(torch.count_nonzero(ws[:flag_bytes])) == 0
