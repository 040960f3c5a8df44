"""bench.py's one-line JSON result, from a short run on one GPU: every key of
the benchmark contract is present with a sensible value (metric and unit, the
whole-job value, the timing fields, the roofline of the dominant kernel, the
end-to-end figure with its host<->device bytes, the clocks sampled during the
timed region, the count of launches of the library's own kernels, and the
per-target figures: each FFN linear from its bf16 activation and the
quantiser per shape, against the measured peaks)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_json_line():
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--steps", "5", "--warmup", "3", "--no-extras",
           "--no-cpu-baseline"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "clocks", "gpu_launches"):
        assert key in d, key
    assert d["unit"] == "TFLOP/s" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["n_gpus"] == 1 and d["steps"] == 5 and d["warmup"] == 3 and d["scaling"] == "weak"
    assert d["data"] == "synthetic" and "workload" in d["config"] and "l2" in d["config"]
    flops = 2.0 * 4096 * 8192 * 2048 + 2.0 * 4096 * 2048 * 8192
    assert d["value"] == pytest.approx(flops / (d["ms_per_step"] * 1e-3) / 1e12, rel=1e-6)
    rf = d["roofline"]
    for key in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert key in rf, key
    assert rf["bound"] == "tensor" and rf["unit"] == "TFLOP/s" and rf["peak"] > 0
    assert rf["frac"] == pytest.approx(rf["achieved"] / rf["peak"], rel=1e-9)
    assert rf["traffic"] is None or rf["traffic"] > 0
    e = d["e2e"]
    assert e["value"] > 0 and e["unit"] == "TFLOP/s"
    assert e["h2d_bytes_per_step"] == 2 * (4096 * 2048 + 4096 * 8192)  # both bf16 activations
    assert e["d2h_bytes_per_step"] == 2 * (4096 * 8192 + 4096 * 2048)  # both bf16 outputs
    c = d["clocks"]
    for key in ("sm_mhz", "sm_max_mhz", "reasons"):
        assert key in c, key
    assert d["gpu_launches"] == 4 * d["steps"]  # two quantisers and two GEMMs per step
    # The per-target figures sit in the last key, so the end of the line carries them.
    assert list(d)[-1] == "targets"
    t = d["targets"]
    for layer in ("ffn_up", "ffn_down"):
        for key in ("linear_us", "linear_tflops", "linear_frac", "quantize_us", "gemm_us", "gemm_frac"):
            assert t[layer][key] > 0, (layer, key)
        M, N, K = (4096, 8192, 2048) if layer == "ffn_up" else (4096, 2048, 8192)
        # (the per-target figures are rounded to four significant digits)
        assert t[layer]["linear_tflops"] == pytest.approx(2.0 * M * N * K / (t[layer]["linear_us"] * 1e-6) / 1e12,
                                                          rel=2e-3)
        assert t[layer]["linear_frac"] == pytest.approx(t[layer]["linear_tflops"] / t["peaks"]["fp8_tflops"], rel=2e-3)
    for key in ("ffn_up_gbs", "ffn_up_frac", "ffn_down_gbs", "ffn_down_frac"):
        assert t["quantizer"][key] > 0, key
    assert rf["linear_ffn_up_frac"] == pytest.approx(t["ffn_up"]["linear_frac"], rel=2e-3)
