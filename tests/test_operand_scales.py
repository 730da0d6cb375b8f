"""The fp16 S-stream's operand scale rule, checked on the host.

pow2_scale_below_2_14(m) (csrc/common.cuh) is the power-of-two scale c that
the fp16 stream applies to S (m = max|S|) and to the iterate (m = max|H|):
c m < 2^14 so no scaled entry reaches the fp16 maximum, c m >= 2^13 so the
largest entries use fp16's top binade (at most 2^63, so that 1/c stays a
normal float), and 1 for m = 0 or a non-finite m.  The header is compiled by
the host compiler into a small shim and called through ctypes.
"""
import ctypes as C
import math
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "symmetric_nmf_clustering_b200", "csrc")
INC = os.path.join(ROOT, "include")
CUDA_INC = "/usr/local/cuda/include"


@pytest.fixture(scope="module")
def scale(tmp_path_factory):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None or not os.path.isdir(CUDA_INC):
        pytest.skip("needs a host C++ compiler and the CUDA headers")
    d = tmp_path_factory.mktemp("scales")
    src = d / "shim.cpp"
    src.write_text('#include "common.cuh"\n'
                   'extern "C" float scale_of(double m) { return symnmf::pow2_scale_below_2_14(m); }\n')
    out = str(d / "libscales.so")
    subprocess.run([cxx, "-O2", "-std=c++17", "-shared", "-fPIC", "-I", CSRC, "-I", INC, "-I", CUDA_INC,
                    str(src), "-o", out], check=True)
    lib = C.CDLL(out)
    lib.scale_of.restype = C.c_float
    lib.scale_of.argtypes = [C.c_double]
    return lib.scale_of


def test_scale_is_a_power_of_two_in_the_top_fp16_binade(scale):
    for m in [1.0, 0.999, 2.0 ** -20, 3.7e-9, 1e-30, 12345.678, 2.0 ** 13, 2.0 ** 14, 1.5 * 2 ** 14,
              3.0e38, 1e-45, 5e-324, 2.0 ** -49, 2.0 ** -50]:
        c = float(scale(m))
        mant, _ = math.frexp(c)
        assert mant == 0.5, (m, c)                     # a power of two
        assert c * m < 2.0 ** 14, (m, c)               # no scaled entry reaches 2^14
        assert c <= 2.0 ** 63, (m, c)                  # 1/c a normal float
        assert c * m >= 2.0 ** 13 or c == 2.0 ** 63, (m, c)   # the top binade unless capped


def test_scale_of_zero_and_non_finite_is_one(scale):
    for m in [0.0, -1.0, math.inf, math.nan]:
        assert scale(m) == 1.0


def test_scale_is_exact_at_powers_of_two(scale):
    # m = 2^e exactly: c = 2^(13 - e), c m = 2^13
    for e in range(-40, 100, 7):
        assert scale(2.0 ** e) == 2.0 ** (13 - e)
