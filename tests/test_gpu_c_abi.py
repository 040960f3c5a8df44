"""The library used from plain C: tests/c_abi_harness.c is compiled with gcc
against include/fp8dit.h and libfp8dit.so (plus the CUDA runtime for device
memory) and run as its own process, with no PyTorch in it. Its weight and
activation codes and scales must equal the oracle's bit for bit, and its
outputs must satisfy the oracle's tolerance."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "dit_rowwise_amax_b200")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


@pytest.fixture(scope="module")
def harness(tmp_path_factory):
    if shutil.which("gcc") is None or not os.path.exists(os.path.join(PKG, "libfp8dit.so")):
        pytest.skip("needs gcc and the built library")
    exe = str(tmp_path_factory.mktemp("harness") / "c_abi_harness")
    cmd = ["gcc", "-O2", "-std=c11", os.path.join(ROOT, "tests", "c_abi_harness.c"),
           "-I" + os.path.join(ROOT, "include"), "-I" + os.path.join(CUDA, "include"),
           "-L" + PKG, "-lfp8dit", "-L" + os.path.join(CUDA, "lib64"), "-lcudart",
           "-Wl,-rpath," + PKG, "-Wl,-rpath," + os.path.join(CUDA, "lib64"), "-o", exe]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return exe


@pytest.mark.parametrize("case", ["tiny", "ragged"])
def test_plain_c_caller(harness, tmp_path, case):
    if case == "tiny":
        d = synth.tiny()
        A, W, bias = d["A"], d["W"], d["bias"]
    else:
        M, N, K = 300, 264, 2064
        A = synth.normal_bf16("gpu/cabi/A", (M, K), 1.0, outlier_p=0.01, outlier_factor=20.0)
        W = synth.normal_bf16("gpu/cabi/W", (N, K), 0.02)
        bias = synth.normal_bf16("gpu/cabi/b", (N,), 0.1)
    M, K = A.shape
    N = W.shape[0]
    for name, arr in (("a.bin", A), ("w.bin", W), ("bias.bin", bias)):
        np.ascontiguousarray(arr, dtype=np.uint16).tofile(str(tmp_path / name))
    r = subprocess.run([harness, str(tmp_path), str(M), str(N), str(K)], capture_output=True, text=True,
                       timeout=120)
    assert r.returncode == 0, r.stderr
    rd = lambda n, dt: np.fromfile(str(tmp_path / n), dtype=dt)
    qw, sw = rd("qw.bin", np.uint8).reshape(N, K), rd("sw.bin", np.float32)
    qa, sa = rd("qa.bin", np.uint8).reshape(M, K), rd("sa.bin", np.float32)
    y = rd("y.bin", np.uint16).reshape(M, N)
    qwo, swo = oracle.quantize_rows(W, oracle.E4M3FN)
    qao, sao = oracle.quantize_rows(A, oracle.E4M3FN)
    assert np.array_equal(qw, qwo) and np.array_equal(sw, swo)
    assert np.array_equal(qa, qao) and np.array_equal(sa, sao)
    ref = oracle.linear(qao, sao, qwo, swo, bias)
    ok, worst = oracle.tolerance_ok(synth.bf16_to_f32(y).astype(np.float64), ref)
    assert ok, f"tolerance exceeded: worst error / bound = {worst:.3f}"
