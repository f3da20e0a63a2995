import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running full-size case")


@pytest.fixture(scope="session")
def cuda_ok():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return True


def pytest_terminal_summary(terminalreporter):
    """Parity figures of the GPU tests: the error the bound is judged on (bf16
    outputs: each |diff| less the half-ulp of the stored value) and the plain
    max |diff| / rms beside it."""
    try:
        from kda_testlib import PARITY_LOG
    except Exception:  # noqa: BLE001 - nothing to report
        return
    if not PARITY_LOG:
        return
    tr = terminalreporter
    tr.write_sep("-", "parity: max|d|/rms judged (plain) <= bound")
    for label, e, raw, tol in PARITY_LOG:
        tr.write_line(f"{label:60s} {e:.3e} ({raw:.3e}) <= {tol:g}")
