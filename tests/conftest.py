import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Per test: the sampler rows compared with the oracle, the kept sets checked
    element by element, and the near-tie / cut-tie rows (allowed exceptions)."""
    try:
        from parity_helpers import REPORT
    except Exception:
        return
    if not REPORT:
        return
    agg = {}
    for name, st in REPORT:
        a = agg.setdefault(name, {})
        for key, v in st.items():
            a[key] = a.get(key, 0) + v
    tr = terminalreporter
    tr.section("sampler parity: rows, kept sets checked, near-ties, cut-ties, allowed token mismatches")
    for name, a in agg.items():
        tr.write_line(f"{name}: rows {a['rows']}, kept {a['kept_checked']}, near-tie {a['near_tie']}, "
                      f"cut-tie {a['cut_tie']}, mismatch {a['mismatch_allowed']}")
