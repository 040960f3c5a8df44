"""The entry points inside a captured CUDA graph: every replay, with new
inputs copied into the captured buffers, gives exactly the eager result for
those inputs. (The benchmark times the FFN step and each kernel this way.)"""
import numpy as np
import pytest
import torch

import synth
from conftest import to_device_bf16

pytestmark = pytest.mark.gpu

fp8 = pytest.importorskip("dit_rowwise_amax_b200")


def capture(fn):
    """Warm fn up on a side stream, then capture one call of it."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t


def check_replays(make_inputs, buffers, run, outputs, n=3):
    """make_inputs(i) -> list of tensors copied into `buffers` before replay i;
    run() reads `buffers` and writes `outputs`; eager results are computed by
    the same run() on the same buffers."""
    g = capture(run)
    for i in range(n):
        for b, x in zip(buffers, make_inputs(i)):
            b.copy_(x)
        torch.cuda.synchronize()
        run()
        torch.cuda.synchronize()
        eager = [o.clone() for o in outputs]
        for o in outputs:
            o.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert fp8.device_error() == 0
        for o, e in zip(outputs, eager):
            assert torch.equal(bits(o), bits(e)), f"replay {i} differs from eager"


def rand_bf16(name, shape, std=1.0):
    return to_device_bf16(synth.normal_bf16(name, shape, std, outlier_p=0.01, outlier_factor=20.0))


def test_quantize_and_linear_step():
    """The benchmark's FFN step pattern: quantise, then the FP8 GEMM from the
    codes; plus the one-call bf16 linear."""
    M, N, K = 1000, 1536, 2064
    W = synth.normal_bf16("gpu/graph/W", (N, K), 0.02)
    layer = fp8.FP8Linear.from_weight(to_device_bf16(W), rand_bf16("gpu/graph/b", (N,), 0.1))
    a = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    qa = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    sa = torch.empty((M,), dtype=torch.float32, device="cuda")
    y1 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    y2 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")

    def run():
        fp8.quantize_rowwise(a, q=qa, scale=sa)
        layer.forward_fp8(qa, sa, y=y1)
        layer.forward(a, y=y2)

    check_replays(lambda i: [rand_bf16(f"gpu/graph/A{i}", (M, K))], [a], run, [qa, sa, y1, y2])


def test_multi_act_weight_only_and_fused():
    M, K = 600, 1024
    layers = [fp8.FP8Linear.from_weight(rand_bf16(f"gpu/graph/W{p}", (n, K), 0.02), None)
              for p, n in (("q", 512), ("k", 256), ("v", 512))]
    a = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    ys = [torch.empty((M, l.N), dtype=torch.bfloat16, device="cuda") for l in layers]
    qa = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    sa = torch.empty((M,), dtype=torch.float32, device="cuda")
    qh = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    sh = torch.empty((M,), dtype=torch.float32, device="cuda")
    yw = torch.empty((M, 512), dtype=torch.bfloat16, device="cuda")
    yf = torch.empty((M, 512), dtype=torch.bfloat16, device="cuda")
    qf = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    sf = torch.empty((M,), dtype=torch.float32, device="cuda")
    fp8.act_quantize_rowwise(a, "gelu")  # builds the activation tables (synchronises once) before capture

    def run():
        fp8.scaled_linear_multi(layers, a, ys=ys, qa_scratch=qa, sa_scratch=sa)
        fp8.act_quantize_rowwise(a, "gelu", q=qh, scale=sh)
        layers[0].forward_weight_only(a, y=yw)
        layers[2].forward_fused(a, y=yf, qa_scratch=qf, sa_scratch=sf)

    check_replays(lambda i: [rand_bf16(f"gpu/graph/B{i}", (M, K))], [a], run, ys + [qh, sh, yw, yf, qf, sf])
