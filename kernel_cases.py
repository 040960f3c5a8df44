"""Run one kernel of the FP8 linear path a few times on the synthetic workload
inputs, for profiling it on its own (for example under Nsight Compute):

    python kernel_cases.py weight_only_ffn_up --iters 4

Cases (inputs from ``synth``, the same as the benchmark's):
    quantize_ffn_up, quantize_ffn_down   rowwise E4M3 quantiser on the FFN activations
    quantize_hidden                      rowwise E4M3 quantiser on hidden_states [32760, 2048]
    gelu_quantize_ffn_down               GELU -> E4M3 producer on a [4096, 8192] activation
    gemm_ffn_up, gemm_ffn_down           FP8 GEMM + epilogue from pre-quantised activations
    weight_only_ffn_up, ..._ffn_down     FP8 weight-only GEMM (bf16 activation)
    fused_ffn_up, fused_ffn_down         the fused linear (one launch: quantise, then GEMM)
    gemm_text_ffn_down                   FP8 GEMM, 26 tokens x FFN-down weight, plain schedule
    split_k_text_ffn_down                the same with a workspace attached (split-K schedule)
    weight_only_text_ffn_down            FP8 weight-only GEMM, 26 tokens x FFN-down weight
    split_k_weight_only_text_ffn_down    the same with a workspace attached (split-K schedule)
    state_dict_e4m3fn, state_dict_e5m2   per-tensor conversion of the 192-tensor DiT weight set
    qkv_encoder                          Q/K/V projections of encoder_hidden_states [26, 2048]:
                                         one quantise + one grouped GEMM (128 x 64 tiles)
    state_dict_e4m3fn_4blocks            the same on the first 4 blocks' 24 tensors (400 MB of bf16,
                                         above L2; small enough for a multi-pass profile)
Layer creation runs the per-channel weight quantiser first; every case then
launches only its own kernels. Exits non-zero if the device reports an error.
"""
import argparse
import os
import sys

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402
from dit_rowwise_amax_b200 import (E4M3FN, E5M2, FP8Linear, act_quantize_rowwise, device_error,  # noqa: E402
                                   quantize_per_tensor, quantize_rowwise, scaled_linear_multi)

CASES = ("quantize_ffn_up", "quantize_ffn_down", "quantize_hidden", "gelu_quantize_ffn_down", "gemm_ffn_up", "gemm_ffn_down",
         "weight_only_ffn_up", "weight_only_ffn_down", "fused_ffn_up", "fused_ffn_down", "gemm_text_ffn_down",
         "split_k_text_ffn_down", "weight_only_text_ffn_down", "split_k_weight_only_text_ffn_down",
         "state_dict_e4m3fn", "state_dict_e5m2", "state_dict_e4m3fn_4blocks", "qkv_encoder")
STATE_DICT_4BLOCKS = 24  # tensors in the first four DiT blocks
TEXT_TOKENS = 26  # encoder_hidden_states length


def _dev(a: np.ndarray, dev) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)


def run(case: str, iters: int) -> None:
    dev = torch.device("cuda", 0)
    if case.startswith("state_dict"):
        layout = synth.state_dict_layout()
        if case.endswith("_4blocks"):
            layout = layout[:STATE_DICT_4BLOCKS]
        tensors = [_dev(synth.state_dict_tensor(n, s), dev) for n, s in layout]
        outs = [torch.empty(t.shape, dtype=torch.uint8, device=dev) for t in tensors]
        scales = torch.empty((len(tensors),), dtype=torch.float32, device=dev)
        fmt = E5M2 if "e5m2" in case else E4M3FN
        for _ in range(iters):
            quantize_per_tensor(tensors, fmt, outs=outs, scales=scales)
        torch.cuda.synchronize()
        if device_error() != 0:
            raise SystemExit(f"{case}: device error word set")
        return
    if case == "qkv_encoder":
        att = synth.attention()
        layers = [FP8Linear.from_weight(_dev(att[f"W_{p}"], dev), _dev(att[f"bias_{p}"], dev)) for p in "qkv"]
        a = _dev(att["encoder"], dev)
        M, K = a.shape
        qa = torch.empty((M, K), dtype=torch.uint8, device=dev)
        sa = torch.empty((M,), dtype=torch.float32, device=dev)
        ys = [torch.empty((M, layer.N), dtype=torch.bfloat16, device=dev) for layer in layers]
        for _ in range(iters):
            scaled_linear_multi(layers, a, ys=ys, qa_scratch=qa, sa_scratch=sa)
        torch.cuda.synchronize()
        if device_error() != 0:
            raise SystemExit(f"{case}: device error word set")
        return
    if case == "quantize_hidden":
        a = _dev(synth.attention()["hidden"], dev)
    else:
        workload = synth.ffn_up() if case.endswith("ffn_up") else synth.ffn_down()
        rows = workload["A"][:TEXT_TOKENS] if "_text_" in case else workload["A"]
        a = _dev(rows, dev)
    M, K = a.shape
    if case.startswith("quantize"):
        q = torch.empty((M, K), dtype=torch.uint8, device=dev)
        s = torch.empty((M,), dtype=torch.float32, device=dev)
        for _ in range(iters):
            quantize_rowwise(a, q=q, scale=s)
    elif case.startswith("gelu_quantize"):
        q = torch.empty((M, K), dtype=torch.uint8, device=dev)
        s = torch.empty((M,), dtype=torch.float32, device=dev)
        for _ in range(iters):
            act_quantize_rowwise(a, "gelu", q=q, scale=s)
    else:
        layer = FP8Linear.from_weight(_dev(workload["W"], dev), _dev(workload["bias"], dev))
        y = torch.empty((M, layer.N), dtype=torch.bfloat16, device=dev)
        op = case[len("split_k_"):] if case.startswith("split_k_") else case
        if op != case:
            layer.attach_workspace()
        if op.startswith("gemm") or op == "text_ffn_down":
            qa, sa = quantize_rowwise(a)
            for _ in range(iters):
                layer.forward_fp8(qa, sa, y=y)
        elif op.startswith("weight_only"):
            for _ in range(iters):
                layer.forward_weight_only(a, y=y)
        else:
            qa = torch.empty((M, layer.K), dtype=torch.uint8, device=dev)
            sa = torch.empty((M,), dtype=torch.float32, device=dev)
            layer.attach_workspace()
            for _ in range(iters):
                layer.forward_fused(a, y=y, qa_scratch=qa, sa_scratch=sa)
    torch.cuda.synchronize()
    if device_error() != 0:
        raise SystemExit(f"{case}: device error word set")


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("case", choices=CASES)
    ap.add_argument("--iters", type=int, default=4)
    args = ap.parse_args(argv)
    run(args.case, args.iters)
    print("ok", args.case)
    return 0


if __name__ == "__main__":
    sys.exit(main())
