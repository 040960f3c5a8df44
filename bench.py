"""Benchmark of the FP8 DiT linear hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fp8dit|reference] [--no-extras]

One step = the two FFN linears of a DiT block at the pages' shapes
("从 BF16 到 FP8：HunyuanVideo1.5推理优化复盘", section 三.2), each the full
path from a bf16 activation (section 三.1):
  FFN-up   A [4096, 2048] -> per-token E4M3 quant -> GEMM vs W [8192, 2048] -> scale/bias/bf16
  FFN-down A [4096, 8192] -> per-token E4M3 quant -> GEMM vs W [2048, 8192] -> scale/bias/bf16
Inputs are synthetic (seeded, see synth/), resident in HBM before timing;
three rotating input/output sets (~0.7 GB) keep every step's operands out of
L2 (126 MB). Timing: CUDA events on the launching stream, W warm-up steps,
K timed steps between a barrier + synchronize on both sides, max over ranks.

`value` = FP8 linear TFLOP/s (2MNK per linear, quantisation time included).
Also reported: the quantiser's HBM GB/s, per-kernel times, a roofline of the
dominant kernel (the GEMM), NVML clocks during the timed region, an
end-to-end figure through the public API with host buffers, and (N=1) the
CPU oracle timed on the host as a baseline. `--impl reference` times the CPU
oracle alone on bounded samples of the same workload.

Under torchrun (N > 1) every rank runs the same per-GPU workload with no
data-path collective (weak scaling); only the timing uses the process group.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "fused FP8 linear TFLOP/s (% FP8 peak) at FFN shapes; quantizer GB/s (% HBM)"
WORKLOAD = "FFN-up 4096x8192x2048 + FFN-down 4096x2048x8192 FP8 linear from bf16 activations"
REFERENCE_BUDGET_S = 120.0  # whole --impl reference run, seconds
E2E_CHUNK_ROWS = 2048  # host-pipeline chunk for the end-to-end measurement
E2E_SLOTS = 2
FFN = (("up", 4096, 8192, 2048), ("down", 4096, 2048, 8192))
FLOPS_PER_STEP = sum(2.0 * M * N * K for _, M, N, K in FFN)
# Quantiser algorithmic bytes: bf16 read + FP8 write + fp32 scale per row.
QBYTES = {name: 2 * M * K + M * K + 4 * M for name, M, N, K in FFN}
FP8_OVER_BF16 = 2.0  # nominal dense ratio (4.5 / 2.25 PFLOP/s)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Idle time before each per-kernel / per-layer region, so that every burst
# figure starts from the same power state as the headline step. Right after
# tens of milliseconds of power-capped GEMMs the power controller holds the
# clocks down for a while: measured on one box, the FFN-up quantiser region
# read 6.2 us and the FFN-down linear region 78 us straight after 27 ms of
# FFN steps, and 5.1 / 69.5 us after 50 ms or more of idle. The loaded state
# is reported separately (targets.sustained).
REST_S = 0.2


def config_dict(n_gpus: int) -> dict:
    return {"workload": WORKLOAD, "a_dist": "up: N(0,1)+0.5% x30; down: GELU(N(0,1))",
            "w_dist": "up N(0,0.02), down N(0,0.015), per-channel E4M3FN", "seed": 0,
            "l2": "3 rotating input/output sets (~0.7 GB > L2)", "parallelism": f"replicas x{n_gpus}"}


# ------------------------------------------------------------------ helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value: float, device=None) -> float:
    """The largest value any rank holds (identity without a process group).
    Timing only: the FP8 path itself exchanges nothing between ranks."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    if device is None:
        device = torch.device("cpu") if dist.get_backend() == "gloo" else torch.device("cuda", torch.cuda.current_device())
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, work_per_step: float, steps: int, max_elapsed_ms: float, scale: float = 1e12) -> float:
    """Units all ranks processed / the slowest rank's time (weak scaling: each
    rank runs the full per-GPU workload)."""
    return world * work_per_step * steps / (max_elapsed_ms * 1e-3) / scale


class ClockSampler:
    """NVML sampling of SM clock and throttle reasons during the timed region."""
    REASONS = {
        "hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
        "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80, "sync_boost": 0x10,
    }

    def __init__(self, torch_device, period_s: float = 0.005):
        self.period = period_s
        self.samples = []
        self.reason_bits = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            import torch
            props = torch.cuda.get_device_properties(torch_device)
            try:  # NVML enumerates physical GPUs; match the CUDA device by UUID
                self._h = pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(props.uuid))
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(torch_device.index or 0)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # reported, not fatal
            self._nvml = None
            self.error = str(e)

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reason_bits |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self) -> dict:
        if self._thread is not None:
            self._stop.set()
            self._thread.join()
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        reasons = [k for k, bit in self.REASONS.items() if self.reason_bits & bit]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples)}


def kernel_source_digest() -> str:
    h = hashlib.sha256()
    for rel in ("dit_rowwise_amax_b200/csrc/gemm_sm100.cu", "dit_rowwise_amax_b200/csrc/fp8dit_internal.cuh"):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d.get(kernel)
        if e and e.get("source_digest") == kernel_source_digest():
            return e.get("bytes_per_launch")
    except (OSError, ValueError):
        pass
    return None


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# ------------------------------------------------------------ CPU oracle leg
def oracle_sample_step(data, rows: int):
    """The oracle on the first `rows` rows of both FFN linears: per-token
    quantisation of A, per-channel of W (prepared once), exact GEMM + epilogue."""
    import oracle
    flops = 0.0
    for name, M, N, K in FFN:
        d = data[name]
        qa, sa = oracle.quantize_rows(d["A"][:rows], oracle.E4M3FN)
        oracle.linear(qa, sa, d["qw"], d["sw"], d["bias"])
        flops += 2.0 * rows * N * K
    return flops


def oracle_data():
    import oracle
    import synth
    data = {"up": synth.ffn_up(), "down": synth.ffn_down()}
    for d in data.values():
        d["qw"], d["sw"] = oracle.quantize_rows(d["W"], oracle.E4M3FN)
    return data


def calibrate_rows(data, target_s: float) -> int:
    import oracle
    probe = max(2, oracle.num_threads())  # the oracle parallelises over rows
    t0 = time.perf_counter()
    oracle_sample_step(data, probe)
    dt = max(time.perf_counter() - t0, 1e-4)
    return int(max(probe, min(4096, probe * target_s / dt)))


def oracle_component_rates(data, rows: int) -> dict:
    """The oracle's parts timed on their own: the exact GEMM per FFN layer on
    all cores, and the quantisers single-threaded and on all cores (GB/s of
    bf16 read + codes written + scales)."""
    import oracle
    import synth
    out = {"gemm_gflops_all_cores": {}, "rowwise_quantiser_gbs": {}, "per_tensor_quantiser_gbs": {}}
    for name, M, N, K in FFN:
        d = data[name]
        qa, sa = oracle.quantize_rows(d["A"][:rows], oracle.E4M3FN)
        t0 = time.perf_counter()
        oracle.linear(qa, sa, d["qw"], d["sw"], d["bias"])
        out["gemm_gflops_all_cores"][f"ffn_{name}"] = 2.0 * rows * N * K / (time.perf_counter() - t0) / 1e9
    hidden = synth.attention()["hidden"][:4096]
    tensor = synth.state_dict_tensor(*synth.state_dict_layout()[4])  # a [8192, 2048] FFN weight
    for threads, label in ((1, "1_thread"), (0, f"{oracle.num_threads()}_threads")):
        oracle.set_threads(threads)
        t0 = time.perf_counter()
        oracle.quantize_rows(hidden, oracle.E4M3FN)
        out["rowwise_quantiser_gbs"][label] = (3 * hidden.size + 4 * hidden.shape[0]) / (time.perf_counter() - t0) / 1e9
        t0 = time.perf_counter()
        oracle.quantize_tensor(tensor, oracle.E4M3FN)
        out["per_tensor_quantiser_gbs"][label] = (3 * tensor.size + 4) / (time.perf_counter() - t0) / 1e9
    oracle.set_threads(0)
    out["samples"] = (f"GEMM: first {rows} rows of each FFN layer; rowwise: hidden_states rows 0..4095 "
                      f"[4096, 2048]; per-tensor: one [8192, 2048] weight")
    return out


def cpu_baseline(target_s: float = 12.0) -> dict:
    import oracle
    data = oracle_data()
    rows = calibrate_rows(data, target_s)
    t0 = time.perf_counter()
    flops = oracle_sample_step(data, rows)
    dt = time.perf_counter() - t0
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"first {rows} rows of both FFN linears (quantise + exact GEMM + epilogue), {dt:.1f} s",
            "cpu": cpu_model(), "components": oracle_component_rates(data, max(16, rows // 4))}


def run_reference(args, world, rank):
    """The CPU oracle as the reference arm: each step one bounded sample."""
    if rank != 0:
        return
    import oracle
    data = oracle_data()
    # Each step is sized so that the whole run (warm-up included) takes about
    # REFERENCE_BUDGET_S, and at most 1.5 s a step.
    per_step_s = min(1.5, REFERENCE_BUDGET_S / (args.steps + args.warmup))
    rows = calibrate_rows(data, per_step_s)
    for _ in range(args.warmup):
        oracle_sample_step(data, rows)
    t0 = time.perf_counter()
    flops = 0.0
    for _ in range(args.steps):
        flops += oracle_sample_step(data, rows)
    dt = time.perf_counter() - t0
    value = flops / dt / 1e12
    sample = f"first {rows} rows of both FFN linears per step (quantise + exact GEMM + epilogue)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64 exact / f64",
        "data": "synthetic", "config": config_dict(world),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample, "cpu": cpu_model()},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU leg
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("fp8dit", "reference"), default="fp8dit")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the attention, state-dict and sustained measurements (and the context file)")
    ap.add_argument("--extras-out", default=None,
                    help="also measure the context figures (library GEMMs, variants, schedules) into this JSON file")
    ap.add_argument("--sustained-s", type=float, default=2.0, help="seconds of back-to-back steps for `sustained`")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_env()

    if args.impl == "reference":
        run_reference(args, world, rank)
        return

    import torch
    import torch.distributed as dist

    import dit_rowwise_amax_b200 as fp8
    import synth

    fp8.load_library()  # fails loudly if the CUDA library is missing
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    def up(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    host = {"up": synth.ffn_up(), "down": synth.ffn_down()}
    layers = {name: fp8.FP8Linear.from_weight(up(host[name]["W"]), up(host[name]["bias"])) for name, *_ in FFN}
    R = 3
    sets = []
    for _ in range(R):
        s = {}
        for name, M, N, K in FFN:
            s[name] = {"A": up(host[name]["A"]),
                       "qa": torch.empty((M, K), dtype=torch.uint8, device=dev),
                       "sa": torch.empty((M,), dtype=torch.float32, device=dev),
                       "y": torch.empty((M, N), dtype=torch.bfloat16, device=dev)}
        sets.append(s)
    torch.cuda.synchronize()

    stream = torch.cuda.current_stream(dev)

    def quantize(name, i):
        b = sets[i % R][name]
        fp8.quantize_rowwise(b["A"], fp8.E4M3FN, q=b["qa"], scale=b["sa"])

    def gemm(name, i):
        b = sets[i % R][name]
        layers[name].forward_fp8(b["qa"], b["sa"], y=b["y"])

    def linear(name, i):  # the whole layer from the bf16 activation: quantiser + GEMM
        b = sets[i % R][name]
        layers[name].forward(b["A"], y=b["y"], qa_scratch=b["qa"], sa_scratch=b["sa"])

    def step(i):
        for name, *_ in FFN:
            quantize(name, i)
            gemm(name, i)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if fp8.device_error(dev) != 0:
        raise RuntimeError("device error during warm-up")

    # Timed region 1 (the headline value): the K steps captured into one CUDA
    # graph (after the W eager warm-up steps), replayed once untimed to upload
    # and warm it, then once timed; only the region is bracketed by events, so
    # consecutive kernels overlap their launch with the predecessor's tail
    # (programmatic dependent launch edges in the graph).
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        step(0)  # a warm-up step on the capture stream
    stream.wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(args.steps):
            step(i)
    graph.replay()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    t_start.record(stream)
    graph.replay()
    t_end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_end), dev)
    if fp8.device_error(dev) != 0:
        raise RuntimeError("device error during the timed region")
    del graph
    # The same K steps launched eagerly from Python, for comparison.
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_start.record(stream)
    for i in range(args.steps):
        step(i)
    t_end.record(stream)
    torch.cuda.synchronize()
    eager_ms = max_over_ranks(t_start.elapsed_time(t_end), dev)

    # Per-kernel and per-layer regions: KR back-to-back launches (or layer
    # calls) on the rotating buffers, captured in a CUDA graph and timed over
    # one replay; consecutive launches overlap launch and tail as in the step,
    # the graph takes the host's per-call launch cost (~8 us from Python) out
    # of the shorter kernels' figures, and KR >= 200 amortises the region's
    # first launch, which has no predecessor to overlap with. Every region
    # starts after REST_S of idle (see REST_S).
    KR = max(args.steps, 200)
    k_avg = {}
    for name, *_ in FFN:
        k_avg[f"quantize_{name}"] = graph_region_ms(torch, lambda i, n=name: quantize(n, i), KR, dev, world)
    peaks, peak_src = load_peaks()
    extras = world == 1 and rank == 0 and not args.no_extras
    q_hidden = measure_hidden_quantizer(fp8, torch, synth, dev, up, peaks["hbm_gbs"]) if extras else {}
    for name, *_ in FFN:
        k_avg[f"gemm_{name}"] = graph_region_ms(torch, lambda i, n=name: gemm(n, i), KR, dev, world)
    # Each FFN layer as a whole (quantiser + GEMM per call), five regions per
    # layer interleaved, the median kept.
    layer_runs = {name: [] for name, *_ in FFN}
    for _ in range(5):
        for name, *_ in FFN:
            layer_runs[name].append(graph_region_ms(torch, lambda i, n=name: linear(n, i), KR, dev, world))
    layer_ms = {name: statistics.median(v) for name, v in layer_runs.items()}
    if fp8.device_error(dev) != 0:
        raise RuntimeError("device error during the per-kernel regions")
    step2_ms = sum(k_avg.values())

    value = whole_job_rate(world, FLOPS_PER_STEP, args.steps, elapsed_ms)
    fp8_peak = peaks["bf16_tflops"] * FP8_OVER_BF16  # burst: every region above lasts milliseconds
    fp8_peak_sustained = peaks["bf16_tflops_sustained"] * FP8_OVER_BF16
    hbm_peak = peaks["hbm_gbs"]

    gemm_us = (k_avg["gemm_up"] + k_avg["gemm_down"]) / 2 * 1e3
    gemm_flops = 2.0 * 4096 * 8192 * 2048
    gemm_tflops = gemm_flops / (gemm_us * 1e-6) / 1e12
    traffic = profiled_traffic("gemm_e4m3_kernel")
    q_gbs = {n: QBYTES[n] / (k_avg[f"quantize_{n}"] * 1e-3) / 1e9 for n in ("up", "down")}
    layer_tf = {n: 2.0 * M * N * K / (layer_ms[n] * 1e-3) / 1e12 for n, M, N, K in FFN}
    roofline = {"bound": "tensor", "kernel": "gemm_e4m3_kernel (FFN-up and FFN-down, mean)",
                "achieved": gemm_tflops, "peak": fp8_peak, "unit": "TFLOP/s", "frac": gemm_tflops / fp8_peak,
                "traffic": traffic,
                "peak_source": f"{peak_src} bf16 burst x {FP8_OVER_BF16:g} (nominal FP8/BF16 ratio)",
                "linear_ffn_up_frac": layer_tf["up"] / fp8_peak, "linear_ffn_down_frac": layer_tf["down"] / fp8_peak,
                "quantizer_ffn_up_frac": q_gbs["up"] / hbm_peak, "quantizer_ffn_down_frac": q_gbs["down"] / hbm_peak}

    # End to end through the public API with pinned host buffers.
    e2e = measure_e2e(fp8, torch, layers, host, dev, args, world)

    targets = {}
    for n, M, N, K in FFN:
        targets[f"ffn_{n}"] = {
            "linear_us": layer_ms[n] * 1e3, "linear_tflops": layer_tf[n], "linear_frac": layer_tf[n] / fp8_peak,
            "linear_us_runs": [v * 1e3 for v in layer_runs[n]],
            "quantize_us": k_avg[f"quantize_{n}"] * 1e3, "gemm_us": k_avg[f"gemm_{n}"] * 1e3,
            "gemm_frac": 2.0 * M * N * K / (k_avg[f"gemm_{n}"] * 1e-3) / 1e12 / fp8_peak}
    targets["quantizer"] = {"ffn_up_gbs": q_gbs["up"], "ffn_up_frac": q_gbs["up"] / hbm_peak,
                            "ffn_down_gbs": q_gbs["down"], "ffn_down_frac": q_gbs["down"] / hbm_peak}
    targets["quantizer"].update(q_hidden)
    context = None
    if extras:
        targets.update(measure_attention_and_state_dict(fp8, torch, synth, dev, up, fp8_peak, hbm_peak))
        targets["sustained"] = measure_sustained(torch, step, args, dev, fp8_peak_sustained)
        if args.extras_out:
            context = measure_context(fp8, torch, synth, dev, up, peaks, fp8_peak)
    targets["peaks"] = {"fp8_tflops": fp8_peak, "fp8_tflops_sustained": fp8_peak_sustained, "hbm_gbs": hbm_peak,
                        "source": peak_src}

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3 (bf16 in/out, fp32 accumulate)",
        "data": "synthetic", "config": config_dict(world),
        "gpu_launches": 4 * args.steps,  # our kernels in timed region 1
        "timing": "K steps in one CUDA graph (captured after the W eager warm-up steps, replayed once untimed, "
                  "then once timed; events at the region ends)",
        "eager_ms_per_step": eager_ms / args.steps, "frac_of_fp8_peak": value / (fp8_peak * world),
        "clocks": clk, "e2e": e2e, "roofline": roofline,
        "kernels_us": {k: round(v * 1e3, 2) for k, v in k_avg.items()},
        "kernels_timing": f"{KR} back-to-back launches per kernel (or layer call) in one CUDA graph replay",
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        cb = cpu_baseline()
        if context is not None:
            context["cpu_baseline_components"] = cb.pop("components")
        else:
            cb.pop("components")
        line["cpu_baseline"] = cb
    line["targets"] = _sig(targets)  # last: the end of the line carries every per-target figure
    if context is not None:
        context["kernels_note"] = (f"per-kernel times: {KR} back-to-back launches of each kernel alone, replayed from a "
                                   f"CUDA graph; their sum {step2_ms * 1e3:.1f} us vs the step's "
                                   f"{elapsed_ms / args.steps * 1e3:.1f} us")
        os.makedirs(os.path.dirname(os.path.abspath(args.extras_out)), exist_ok=True)
        with open(args.extras_out, "w") as f:
            json.dump(context, f, indent=1)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def _sig(x, digits=4):
    """x with every float rounded to `digits` significant digits (a shorter line)."""
    if isinstance(x, dict):
        return {k: _sig(v, digits) for k, v in x.items()}
    if isinstance(x, list):
        return [_sig(v, digits) for v in x]
    if isinstance(x, float) and x != 0.0 and np.isfinite(x):
        return float(f"{x:.{digits}g}")
    return x


def measure_sustained(torch, step, args, dev, fp8_peak_sustained, n_steps=200):
    """The step, back to back for at least --sustained-s seconds (a graph of
    n_steps steps replayed repeatedly), with NVML clocks sampled meanwhile: the
    regime a denoising loop runs in, against the sustained peak."""
    cur = torch.cuda.current_stream(dev)
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(dev)
    side.wait_stream(cur)
    with torch.cuda.stream(side):
        step(0)
    cur.wait_stream(side)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        for i in range(n_steps):
            step(i)
    g.replay()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(cur)
    g.replay()
    b.record(cur)
    torch.cuda.synchronize()
    reps = max(1, int(args.sustained_s / max(a.elapsed_time(b) * 1e-3, 1e-6) + 0.5))
    clocks = ClockSampler(dev, period_s=0.01)
    clocks.start()
    a.record(cur)
    for _ in range(reps):
        g.replay()
    b.record(cur)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = a.elapsed_time(b)
    del g
    tf = FLOPS_PER_STEP * n_steps * reps / (ms * 1e-3) / 1e12
    return {"seconds": ms * 1e-3, "steps": n_steps * reps, "tflops": tf, "frac": tf / fp8_peak_sustained,
            "sm_mhz": clk["sm_mhz"], "reasons": clk["reasons"], "clock_samples": clk["samples"]}


def measure_e2e(fp8, torch, layers, host, dev, args, world):
    """Same metric through the host-buffer API (FP8Linear.forward_host ->
    fp8_scaled_linear_host): every step copies both activations host->device
    from pinned memory and both outputs device->host, chunk by chunk,
    overlapped with the kernels and with each other by the library's
    pipeline; the step ends when the last output row has reached host memory."""
    pinned = {}
    for name, M, N, K in FFN:
        a = torch.from_numpy(np.ascontiguousarray(host[name]["A"]).view(np.int16)).view(torch.bfloat16)
        pinned[name] = {"A": a.pin_memory(), "y": torch.empty((M, N), dtype=torch.bfloat16).pin_memory()}
        layers[name].attach_host_pipeline(chunk_rows=E2E_CHUNK_ROWS, slots=E2E_SLOTS)
    h2d = sum(2 * M * K for _, M, N, K in FFN)
    d2h = sum(2 * M * N for _, M, N, K in FFN)
    stream = torch.cuda.current_stream(dev)

    def step():
        for name, *_ in FFN:
            p = pinned[name]
            layers[name].forward_host(p["A"], y=p["y"])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    steps = max(1, min(args.steps, 50))
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0.record(stream)
    for _ in range(steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), dev)
    for name, *_ in FFN:
        layers[name].detach_host_pipeline()
    return {"value": whole_job_rate(world, FLOPS_PER_STEP, steps, ms), "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "api": f"FP8Linear.forward_host (fp8_scaled_linear_host: chunks of {E2E_CHUNK_ROWS} rows, "
                   f"{E2E_SLOTS} slots, copy-in / quantise + GEMM / copy-out overlapped) from pinned host memory"}


def rest(torch):
    """Let the GPU idle for REST_S before a burst region."""
    torch.cuda.synchronize()
    time.sleep(REST_S)


def graph_region_ms(torch, fn, n, dev, world=1, warm=3):
    """Device time per call of n back-to-back calls of fn, captured into one
    CUDA graph and replayed (once untimed, to upload and warm it; then once
    timed, events at the ends; max over ranks), after REST_S of idle.
    Replaying removes the host's per-call launch cost, which exceeds the
    device time of the smaller kernels."""
    rest(torch)
    cur = torch.cuda.current_stream(dev)
    side = torch.cuda.Stream(dev)
    side.wait_stream(cur)
    with torch.cuda.stream(side):
        for i in range(warm):
            fn(i)
    cur.wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(n):
            fn(i)
    g.replay()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    a.record(cur)
    g.replay()
    b.record(cur)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), dev) if world > 1 else a.elapsed_time(b)
    del g
    return ms / n


def time_region(torch, fn, iters, dev, warm=3):
    """Device time per call of iters eager calls of fn, after REST_S of idle."""
    rest(torch)
    stream = torch.cuda.current_stream(dev)
    for i in range(warm):
        fn(i)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(iters):
        fn(i)
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / iters


def scaled_mm_context(torch, layer, qs, ys, M, N, K, dev):
    """torch._scaled_mm on the layer's E4M3 codes ("rowwise": the per-token
    and per-channel scales of the method; "tensorwise": unit scales, a
    cheaper epilogue than the method needs), timed eagerly over 50 calls
    (each call is longer than the host's launch cost). Records the error
    instead of a time where this torch build refuses a scaling mode; the
    row-scaled result is also compared with the layer's own output."""
    res = {}
    fa = [q.view(torch.float8_e4m3fn) for q, _ in qs]
    fw = layer.qw.view(torch.float8_e4m3fn).t()  # [K, N], column-major
    modes = {"rowwise": ([s.view(M, 1) for _, s in qs], layer.sw.view(1, N)),
             "tensorwise": ([torch.ones((), dtype=torch.float32, device=dev)] * len(qs),
                            torch.ones((), dtype=torch.float32, device=dev))}
    for mode, (sas, sw) in modes.items():
        try:
            run = lambda i: torch._scaled_mm(fa[i % len(fa)], fw, scale_a=sas[i % len(fa)], scale_b=sw,
                                             out_dtype=torch.bfloat16)
            run(0)  # surfaces a refused mode before timing
            ms = time_region(torch, run, 50, dev)
            r = {"us": ms * 1e3, "tflops": 2.0 * M * N * K / (ms * 1e-3) / 1e12}
            if mode == "rowwise":
                # Same quantity up to the bias and two bf16 roundings.
                layer.forward_fp8(qs[0][0], qs[0][1], y=ys[0])
                torch.cuda.synchronize()
                b = layer.bias.float().view(1, N) if layer.bias is not None else 0.0
                r["max_abs_diff_vs_fp8dit"] = (run(0).float() + b - ys[0].float()).abs().max().item()
                r["max_abs_fp8dit"] = ys[0].float().abs().max().item()
            res[mode] = r
        except Exception as e:  # a scaling mode this torch build does not offer
            res[mode] = {"unavailable": f"{type(e).__name__}: {str(e).splitlines()[0][:160]}"}
    return res


def measure_hidden_quantizer(fp8, torch, synth, dev, up, hbm_peak, n=50):
    """The rowwise quantiser on hidden_states [32760, 2048] (two rotating
    inputs, 268 MB > L2), n back-to-back launches replayed from a CUDA graph."""
    att = synth.attention()
    A = [up(att["hidden"]) for _ in range(2)]
    M = att["hidden"].shape[0]
    qa = torch.empty((M, 2048), dtype=torch.uint8, device=dev)
    sa = torch.empty((M,), dtype=torch.float32, device=dev)
    qms = graph_region_ms(torch, lambda i: fp8.quantize_rowwise(A[i % 2], q=qa, scale=sa), n, dev)
    qb = 3 * M * 2048 + 4 * M
    return {"hidden_us": qms * 1e3, "hidden_gbs": qb / (qms * 1e-3) / 1e9, "hidden_frac": qb / (qms * 1e-3) / 1e9 / hbm_peak}


def measure_attention_and_state_dict(fp8, torch, synth, dev, up, fp8_peak, hbm_peak):
    """The target figures beyond the FFN step: the Q / K / V projections (one quantisation
    feeding one grouped launch, HunyuanVideo page section 三.4) on
    hidden_states and encoder_hidden_states, and the merged N = 6144
    alternative; the per-tensor conversion of the 192-tensor weight set."""
    out = {"qkv": {}, "state_dict": {}}
    att = synth.attention()
    layers = [fp8.FP8Linear.from_weight(up(att[f"W_{p}"]), up(att[f"bias_{p}"])) for p in "qkv"]
    # encoder_hidden_states first: its ~10 us launches are latency-bound and
    # read slower in the power state the hidden_states projections leave.
    for name in ("encoder", "hidden"):
        A = [up(att[name]) for _ in range(2)]
        M = att[name].shape[0]
        qa = torch.empty((M, 2048), dtype=torch.uint8, device=dev)
        sa = torch.empty((M,), dtype=torch.float32, device=dev)
        ys = [[torch.empty((M, 2048), dtype=torch.bfloat16, device=dev) for _ in range(3)] for _ in range(2)]
        ms = graph_region_ms(torch, lambda i: fp8.scaled_linear_multi(layers, A[i % 2], ys=ys[i % 2], qa_scratch=qa,
                                                                  sa_scratch=sa), 50, dev)
        flops = 3 * 2.0 * M * 2048 * 2048
        out["qkv"][f"{name}_us"] = ms * 1e3
        out["qkv"][f"{name}_frac"] = flops / (ms * 1e-3) / 1e12 / fp8_peak
    # Merged Q/K/V projection (one N = 6144 GEMM) vs the three separate,
    # grouped projections above, on hidden_states (HunyuanVideo page §三.4).
    A = [up(att["hidden"]) for _ in range(2)]
    M = att["hidden"].shape[0]
    w_qkv = np.concatenate([att["W_q"], att["W_k"], att["W_v"]], axis=0)
    b_qkv = np.concatenate([att["bias_q"], att["bias_k"], att["bias_v"]], axis=0)
    merged = fp8.FP8Linear.from_weight(up(w_qkv), up(b_qkv))
    qa = torch.empty((M, 2048), dtype=torch.uint8, device=dev)
    sa = torch.empty((M,), dtype=torch.float32, device=dev)
    ym = [torch.empty((M, 6144), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    ms = graph_region_ms(torch, lambda i: merged.forward(A[i % 2], y=ym[i % 2], qa_scratch=qa, sa_scratch=sa), 50, dev)
    out["qkv"]["hidden_merged_n6144_us"] = ms * 1e3
    del A, ym, merged, layers
    # State-dict conversion: 192 tensors, 1.61e9 elements, both formats.
    layout = synth.state_dict_layout()
    tensors = [up(synth.state_dict_tensor(n, sh)) for n, sh in layout]
    outs = [torch.empty(t.shape, dtype=torch.uint8, device=dev) for t in tensors]
    scales = torch.empty((len(tensors),), dtype=torch.float32, device=dev)
    numel = sum(t.numel() for t in tensors)
    alg_bytes = 3 * numel + 4 * len(tensors)
    for fmt, fname in ((fp8.E4M3FN, "e4m3fn"), (fp8.E5M2, "e5m2")):
        ms = time_region(torch, lambda i: fp8.quantize_per_tensor(tensors, fmt, outs=outs, scales=scales), 5, dev,
                         warm=2)
        out["state_dict"][f"{fname}_us"] = ms * 1e3
        out["state_dict"][f"{fname}_gbs"] = alg_bytes / (ms * 1e-3) / 1e9
        out["state_dict"][f"{fname}_frac"] = alg_bytes / (ms * 1e-3) / 1e9 / hbm_peak
    del tensors, outs
    return out


def measure_context(fp8, torch, synth, dev, up, peaks, fp8_peak):
    """Context figures, written to the --extras-out file: producer fusion,
    GEMM-only times, the fused (one-launch) linear, the FP8 weight-only path,
    BF16 and library FP8 GEMMs on the same shapes, stream-K and split-K."""
    out = {}
    # Producer fusion (HunyuanVideo page §三.5): FFN-down fed by GELU(h), h the
    # FFN-up output. Fused: one kernel emits (FP8, scale). Unfused: torch's
    # bf16 GELU, then the rowwise quantiser. Both then run the FFN-down GEMM.
    du, dd = synth.ffn_up(), synth.ffn_down()
    lu = fp8.FP8Linear.from_weight(up(du["W"]), up(du["bias"]))
    ld = fp8.FP8Linear.from_weight(up(dd["W"]), up(dd["bias"]))
    hs = [lu.forward(up(du["A"])) for _ in range(2)]  # [4096, 8192] bf16
    qd = torch.empty((4096, 8192), dtype=torch.uint8, device=dev)
    sd = torch.empty((4096,), dtype=torch.float32, device=dev)
    yd = torch.empty((4096, 2048), dtype=torch.bfloat16, device=dev)

    def fused(i):
        fp8.act_quantize_rowwise(hs[i % 2], "gelu", q=qd, scale=sd)
        ld.forward_fp8(qd, sd, y=yd)

    def unfused(i):
        g = torch.nn.functional.gelu(hs[i % 2])
        fp8.quantize_rowwise(g, q=qd, scale=sd)
        ld.forward_fp8(qd, sd, y=yd)

    f_ms = graph_region_ms(torch, fused, 50, dev)
    u_ms = graph_region_ms(torch, unfused, 50, dev)
    a_ms = graph_region_ms(torch, lambda i: fp8.act_quantize_rowwise(hs[i % 2], "gelu", q=qd, scale=sd), 50, dev)
    out["producer_fusion_ffn_down"] = {"fused_us": f_ms * 1e3, "unfused_torch_gelu_us": u_ms * 1e3,
                                       "gelu_quantize_us": a_ms * 1e3,
                                       "gelu_quantize_gbs": 3 * 4096 * 8192 / (a_ms * 1e-3) / 1e9}
    del hs

    # GEMM only (pre-quantised activations) at the FFN shapes.
    for name, M, N, K in FFN:
        d = synth.ffn_up() if name == "up" else synth.ffn_down()
        layer = fp8.FP8Linear.from_weight(up(d["W"]), up(d["bias"]))
        qs = [fp8.quantize_rowwise(up(d["A"])) for _ in range(3)]
        ys = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(3)]
        ms = graph_region_ms(torch, lambda i: layer.forward_fp8(qs[i % 3][0], qs[i % 3][1], y=ys[i % 3]), 100, dev)
        tf = 2.0 * M * N * K / (ms * 1e-3) / 1e12
        out[f"gemm_only_ffn_{name}"] = {"us": ms * 1e3, "tflops": tf, "frac_of_fp8_peak": tf / fp8_peak,
                                        "plan": list(layer.plan(M))}
        # The fused linear (one launch: quantise, then GEMM) against quantiser
        # + GEMM (two launches), both from bf16 A, 100 calls each.
        qa_s = torch.empty((M, K), dtype=torch.uint8, device=dev)
        sa_s = torch.empty((M,), dtype=torch.float32, device=dev)
        a16s = [up(d["A"]) for _ in range(3)]
        uf_ms = graph_region_ms(torch, lambda i: layer.forward(a16s[i % 3], y=ys[i % 3], qa_scratch=qa_s, sa_scratch=sa_s),
                                100, dev)
        fz_ms = graph_region_ms(torch, lambda i: layer.forward_fused(a16s[i % 3], y=ys[i % 3], qa_scratch=qa_s,
                                                                     sa_scratch=sa_s), 100, dev)
        layer.detach_workspace()
        out[f"fused_linear_ffn_{name}"] = {"fused_us": fz_ms * 1e3, "quantizer_plus_gemm_us": uf_ms * 1e3,
                                           "tflops": 2.0 * M * N * K / (fz_ms * 1e-3) / 1e12,
                                           "frac_of_fp8_peak": 2.0 * M * N * K / (fz_ms * 1e-3) / 1e12 / fp8_peak}
        del a16s, qa_s, sa_s
        # FP8 weight-only (bf16 activation, E4M3 weight decoded in shared
        # memory, BF16 tensor cores), same layer.
        a16s = [up(d["A"]) for _ in range(3)]
        wms = graph_region_ms(torch, lambda i: layer.forward_weight_only(a16s[i % 3], y=ys[i % 3]), 100, dev)
        wtf = 2.0 * M * N * K / (wms * 1e-3) / 1e12
        out[f"weight_only_ffn_{name}"] = {"us": wms * 1e3, "tflops": wtf,
                                          "frac_of_bf16_peak": wtf / peaks["bf16_tflops"]}
        del a16s
        # BF16 context: the same shape through torch.matmul (cuBLAS), bench script only.
        a16 = up(d["A"])
        w16 = up(d["W"])
        bms = time_region(torch, lambda i: torch.matmul(a16, w16.t()), 50, dev)
        btf = 2.0 * M * N * K / (bms * 1e-3) / 1e12
        out[f"bf16_torch_matmul_ffn_{name}"] = {"us": bms * 1e3, "tflops": btf}
        # FP8 library context: the same codes through torch._scaled_mm, bf16 out,
        # no bias; bench script only. With per-row / per-column scales torch
        # runs its own CUTLASS sm100 kernel; with one scale per operand, cuBLASLt.
        out[f"fp8_torch_scaled_mm_ffn_{name}"] = scaled_mm_context(torch, layer, qs, ys, M, N, K, dev)
        del a16, w16, qs, ys
    # Stream-K against the tile-per-pair schedule where the latter's last wave
    # is nearly empty: 4864 tokens x FFN-down weight = 152 tiles on 74 pairs.
    d = synth.ffn_down()
    M, N, K = 4864, 2048, 8192
    layer = fp8.FP8Linear.from_weight(up(d["W"]), up(d["bias"]))
    qs = [fp8.quantize_rowwise(up(synth.normal_bf16(f"bench/sk/A{i}", (M, K), 1.0, outlier_p=0.001,
                                                        outlier_factor=20.0))) for i in range(3)]
    ys = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(3)]
    run = lambda i: layer.forward_fp8(qs[i % 3][0], qs[i % 3][1], y=ys[i % 3])
    dp_ms = graph_region_ms(torch, run, 100, dev)
    layer.attach_workspace()
    sk_ms = graph_region_ms(torch, run, 100, dev)
    layer.detach_workspace()
    out["stream_k_4864x2048x8192"] = {"tiles": 152, "pairs": 74, "plain_us": dp_ms * 1e3, "stream_k_us": sk_ms * 1e3,
                                      "stream_k_tflops": 2.0 * M * N * K / (sk_ms * 1e-3) / 1e12,
                                      "speedup": dp_ms / sk_ms}
    del qs, ys, layer
    # Split-K against the plain schedule for few tokens through the FFN-down
    # weight: [M, 8192] x [2048, 8192], 16 tiles of 128 x 128 (M = 26: the
    # encoder_hidden_states length).
    for M in (1, 26, 128):
        layer = fp8.FP8Linear.from_weight(up(d["W"]), up(d["bias"]))
        qs = [fp8.quantize_rowwise(up(synth.normal_bf16(f"bench/split/A{i}", (M, K), 1.0))) for i in range(3)]
        ys = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(3)]
        run = lambda i: layer.forward_fp8(qs[i % 3][0], qs[i % 3][1], y=ys[i % 3])
        a16s = [up(synth.normal_bf16(f"bench/split/A16_{i}", (M, K), 1.0)) for i in range(3)]
        run_wo = lambda i: layer.forward_weight_only(a16s[i % 3], y=ys[i % 3])
        dp_ms = graph_region_ms(torch, run, 200, dev)
        wo_ms = graph_region_ms(torch, run_wo, 200, dev)
        layer.attach_workspace()
        plan = list(layer.plan(M))
        sp_ms = graph_region_ms(torch, run, 200, dev)
        wos_ms = graph_region_ms(torch, run_wo, 200, dev)
        layer.detach_workspace()
        out[f"split_k_{M}x2048x8192"] = {"plain_us": dp_ms * 1e3, "split_k_us": sp_ms * 1e3, "split_plan": plan,
                                         "speedup": dp_ms / sp_ms, "w_gbs_split": N * K / (sp_ms * 1e-3) / 1e9,
                                         "weight_only_plain_us": wo_ms * 1e3,
                                         "weight_only_split_k_us": wos_ms * 1e3,
                                         "weight_only_speedup": wo_ms / wos_ms}
    del qs, ys, layer, a16s
    return out


if __name__ == "__main__":
    main()
