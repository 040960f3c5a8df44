"""The C-ABI library builds for sm_100a, loads without a GPU, and exports
every entry point include/fp8dit.h declares (no compute calls here)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8dit.h")


def declared_functions():
    text = open(HEADER, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s+(fp8[a-z_0-9]*)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def libpath():
    from dit_rowwise_amax_b200 import build
    return build.build()


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ("fp8_quantize_rowwise", "fp8_quantize_weight_per_channel", "fp8_quantize_weight_per_tensor",
                     "fp8_scaled_linear", "fp8_scaled_linear_multi", "fp8_linear_create", "fp8_linear_destroy",
                     "fp8dit_device_error", "fp8dit_last_error_string"):
        assert required in names


def test_library_exports_every_declared_symbol(libpath):
    lib = ctypes.CDLL(libpath)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_library_has_no_oracle_or_torch_dependency(libpath):
    out = subprocess.run(["ldd", libpath], capture_output=True, text=True).stdout
    assert "torch" not in out and "oracle" not in out and "python" not in out
    syms = subprocess.run(["nm", "-D", "--defined-only", libpath], capture_output=True, text=True).stdout
    assert " or_" not in syms


def test_built_for_sm100a_only():
    from dit_rowwise_amax_b200 import build
    flags = " ".join(build.NVCC_FLAGS)
    assert "arch=compute_100a,code=sm_100a" in flags
    assert "use_fast_math" not in flags


def test_header_is_plain_c(tmp_path):
    """include/fp8dit.h in a C11 translation unit (the plain-C caller used by
    the GPU tests), compiled without linking."""
    import shutil
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    if shutil.which("gcc") is None or not os.path.exists(os.path.join(cuda_inc, "cuda_runtime.h")):
        pytest.skip("needs gcc and the CUDA headers")
    r = subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-c", os.path.join(ROOT, "tests", "c_abi_harness.c"),
                        "-I" + os.path.join(ROOT, "include"), "-I" + cuda_inc, "-o", str(tmp_path / "h.o")],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
