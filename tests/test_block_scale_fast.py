"""The quantisers' division-free block scale, checked on the CPU.

The block scale is sb = E4M3(RN(RN(amax_b / 6) / s_t)) (aisight.pl, section
"Architektura NVFP4 kontra ograniczenia mikroskalowania": an E4M3 scale per
16-element block under an FP32 tensor scale; the constant 6 is E2M1's largest
value).  The kernels replace both IEEE divisions with Markstein's correction
step (one multiply by RN(1/b) and two FMAs), clamp the second numerator to
s_t * 2^10, and take this path only for tensor scales in [2^-80, 2^100].
tests/helpers/block_scale_fast.c restates those steps in C; this file checks
them against IEEE division: exhaustively for amax / 6 over every binary32 from
2^-125 up, and for the whole quotient over strided sweeps of every amax at
tensor scales across the fast range, dense where the E4M3 code is decided.
The GPU parity tests then check the kernels' scale bytes bit for bit.
"""
import ctypes as C
import os
import subprocess

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "helpers", "block_scale_fast.c")


@pytest.fixture(scope="module")
def lib(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("bsf") / "libbsf.so")
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
                           "-o", out, SRC, "-lm"])
    L = C.CDLL(out)
    L.div6_mismatches.argtypes = [C.c_uint32, C.c_uint32, C.c_uint32]
    L.div6_mismatches.restype = C.c_int64
    L.t2_mismatches.argtypes = [C.c_float, C.c_uint32, C.c_uint32, C.c_uint32]
    L.t2_mismatches.restype = C.c_int64
    return L


def bits(x):
    return int(np.float32(x).view(np.uint32))


FLT_MAX_BITS = 0x7F7FFFFF


def test_div6_exhaustive_from_2_pow_minus_125(lib):
    assert lib.div6_mismatches(bits(2.0 ** -125), FLT_MAX_BITS, 1) == 0
    # below that the residual underflows and the step is no longer exact: the
    # kernels rely on such quotients giving sb = 0 (next test), not on exactness
    assert lib.div6_mismatches(1, bits(2.0 ** -125) - 1, 1) > 0


TENSOR_SCALES = [2.0 ** -80, 1.37 * 2.0 ** -80, 1.0 / 2688.0, 3.7e-4, 0.0123, 5.96e-8, 1.0, 7.25, 2.5e5,
                 3.1e20, 2.0 ** 99.7, 2.0 ** 100]


@pytest.mark.parametrize("s_t", TENSOR_SCALES)
def test_block_scale_quotient_strided(lib, s_t):
    s_t = float(np.float32(s_t))
    assert lib.t2_mismatches(s_t, 0, FLT_MAX_BITS, 1009) == 0
    # every amax whose quotient lands near the E4M3 range, densely
    lo = bits(np.float32(s_t) * np.float32(6.0 * 2.0 ** -13))
    hi = min(bits(np.float32(s_t) * np.float32(6.0 * 2.0 ** 11)), FLT_MAX_BITS)
    assert lib.t2_mismatches(s_t, lo, hi, 7) == 0


@pytest.mark.parametrize("s_t", [1.0 / 2688.0, 2.0 ** -80])
def test_block_scale_quotient_dense(lib, s_t):
    """Every amax in the window where the quotient decides the code."""
    s_t = float(np.float32(s_t))
    lo = bits(np.float32(s_t) * np.float32(6.0 * 2.0 ** -13))
    hi = bits(np.float32(s_t) * np.float32(6.0 * 2.0 ** 11))
    assert lib.t2_mismatches(s_t, lo, hi, 1) == 0
