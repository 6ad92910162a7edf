"""The sampler's fast quotient x = fl(l / T) (Markstein's method, vsl_math.cuh,
used for rows whose T lies in [2^-20, 2^20] and whose nonzero |l| lie in
[2^-60, 2^100]) against CUDA's IEEE round-to-nearest division, bit for bit,
over every float32 bit pattern of l in that domain (both signs; zeros of
either sign count as zero) for temperatures of every significand shape across
the range and at its edges."""
import ctypes
import os

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TEST_LIB = os.path.join(ROOT, "tests", "libvsl_test.so")


def _temperatures():
    rng = np.random.default_rng(2024)
    sig = [1.0, 1.5, 1.25, float(np.float32(2.0) - np.float32(2.0 ** -23)), 1.0 + 2.0 ** -23]
    sig += rng.uniform(1.0, 2.0, 6).tolist()
    Ts = [s * 2.0 ** e for e in range(-20, 20, 2) for s in sig]
    Ts += rng.uniform(0.05, 1.6, 24).tolist()           # the configurations' temperatures
    Ts += [2.0 ** -20, 2.0 ** 20, float(np.float32(2.0 ** 20) * np.float32(1 - 2.0 ** -24))]
    return np.array(Ts, np.float32)


def test_quotient_matches_ieee_division_on_every_bit_pattern(cuda_device):
    if not os.path.exists(TEST_LIB):
        pytest.fail("tests/libvsl_test.so not built (vocab_sharded_logits_b200/build.py builds it)")
    L = ctypes.CDLL(TEST_LIB)
    L.vsl_test_div_mismatches.restype = ctypes.c_int
    L.vsl_test_div_mismatches.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_uint32, ctypes.c_uint32,
                                          ctypes.POINTER(ctypes.c_ulonglong), ctypes.POINTER(ctypes.c_ulonglong)]
    Ts = _temperatures()
    for lo, hi in ((0x00000000, 0x7FFFFFFF), (0x80000000, 0xFFFFFFFF)):
        count, first = ctypes.c_ulonglong(0), ctypes.c_ulonglong(0)
        st = L.vsl_test_div_mismatches(Ts.ctypes.data, len(Ts), lo, hi, ctypes.byref(count), ctypes.byref(first))
        assert st == 0
        if count.value:
            ti, bits = first.value >> 32, first.value & 0xFFFFFFFF
            l = np.array([bits], np.uint32).view(np.float32)[0]
            pytest.fail(f"{count.value} mismatches; first: l = {l!r} (0x{bits:08x}), T = {Ts[ti]!r}")
