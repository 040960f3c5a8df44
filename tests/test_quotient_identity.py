"""The quantisers' corrected-reciprocal quotient equals IEEE fp32 division
wherever the FP8 code can depend on it: exhaustive over every (bf16 x, bf16
amax) pair with |x| <= amax, for E4M3FN and E5M2 (CPU, C fmaf)."""
import ctypes
import os
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def lib(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("qid") / "libqid.so")
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off",
                           os.path.join(HERE, "quotient_identity.c"), "-o", out, "-lm"])
    L = ctypes.CDLL(out)
    L.quotient_identity_check.restype = ctypes.c_longlong
    L.quotient_identity_check.argtypes = [ctypes.c_float, ctypes.c_float, ctypes.POINTER(ctypes.c_longlong)]
    return L


@pytest.mark.parametrize("fmax,zero_below", [(448.0, 2.0 ** -10), (57344.0, 2.0 ** -17)], ids=["e4m3fn", "e5m2"])
def test_exhaustive(lib, fmax, zero_below):
    differ = ctypes.c_longlong()
    bad = lib.quotient_identity_check(fmax, zero_below, ctypes.byref(differ))
    assert bad == 0, f"{bad} pairs would encode differently ({differ.value} fp32 differences)"
