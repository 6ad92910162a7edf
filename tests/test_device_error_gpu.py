"""The bounded waits' failure report, exercised without a fault: the test
library's probe kernel waits, with a short limit, on an mbarrier nothing ever
arrives at (no copy in flight, no other thread involved), gives up, sets its
site bit in the library's device error word and returns.  vsl_device_error
must report that bit once, clear it, and leave the context usable.  Plus both
entry points called after a device round trip (the per-device launch state)."""
import ctypes
import os

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TEST_LIB = os.path.join(ROOT, "tests", "libvsl_test.so")


def _lib():
    if not os.path.exists(TEST_LIB):
        pytest.fail("tests/libvsl_test.so not built (vocab_sharded_logits_b200/build.py builds it)")
    L = ctypes.CDLL(TEST_LIB)
    L.vsl_test_wait_probe.restype = ctypes.c_int
    L.vsl_test_wait_probe.argtypes = [ctypes.c_longlong, ctypes.c_int, ctypes.c_void_p]
    L.vsl_test_probe_site.restype = ctypes.c_uint32
    L.vsl_device_error.restype = ctypes.c_int
    L.vsl_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32)]
    return L


def _device_error(L):
    code = ctypes.c_uint32(0)
    st = L.vsl_device_error(ctypes.byref(code))
    return st, code.value


def test_wait_that_runs_out_is_reported_and_cleared(cuda_device):
    torch.cuda.init()
    L = _lib()
    assert _device_error(L) == (0, 0)
    site = L.vsl_test_probe_site()
    assert site != 0 and site & (site - 1) == 0
    # about 1 ms at B200 clocks: the wait gives up
    assert L.vsl_test_wait_probe(2_000_000, 0, None) == 0
    st, code = _device_error(L)
    assert st == 6 and code == site            # VSL_ERR_DEVICE_TIMEOUT, the probe's site
    assert _device_error(L) == (0, 0)          # read once, then cleared
    # a wait whose barrier completes reports nothing
    assert L.vsl_test_wait_probe(2_000_000, 1, None) == 0
    assert _device_error(L) == (0, 0)
    # the context is still usable
    x = torch.arange(1024, device=cuda_device, dtype=torch.float32)
    assert float(x.sum().item()) == 1023 * 1024 / 2


def test_invalid_probe_limit_is_rejected_on_the_host(cuda_device):
    L = _lib()
    assert L.vsl_test_wait_probe(0, 0, None) == 1
    assert L.vsl_test_wait_probe(5_000_000_000, 0, None) == 1


def test_entry_points_after_a_device_round_trip(cuda_device):
    """Both calls on cuda:0 with the device made current again after another
    current-device switch, reproducing the first call's results bitwise."""
    import vocab_sharded_logits_b200 as vsl
    import workloads as W
    w = W.scaled(W.WORKLOADS["decode"], V=4 * 2048, requests=16, H=256)
    hidden, ws = W.gemm_inputs(w, cuda_device)
    T, k, p, req, pos = W.row_params(w)
    prm = vsl.make_row_params(T, k, p, req, pos, cuda_device)

    def run():
        lg = vsl.logits_local(hidden, ws)
        out = vsl.sample(lg, prm, 9, w.n_logprobs, kept_theta=True)
        torch.cuda.synchronize()
        return [t.cpu().numpy() for t in lg] + [out.token_ids.cpu().numpy(), out.kept_theta.cpu().numpy()]

    first = run()
    for d in range(torch.cuda.device_count()):
        torch.cuda.set_device(d)
    torch.cuda.set_device(0)
    with torch.cuda.device(0):
        again = run()
    for a, b in zip(first, again):
        assert np.array_equal(a, b, equal_nan=True)
    assert vsl.device_error() == (0, 0)
