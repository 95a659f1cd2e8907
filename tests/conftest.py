import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built library")
    config.addinivalue_line("markers", "slow: full-size CPU oracle runs")


@pytest.fixture(scope="session")
def cuda_available():
    import torch
    return torch.cuda.is_available()


def pytest_terminal_summary(terminalreporter):
    """Prints the error margin of every GPU parity comparison of the run."""
    try:
        from parity import MARGINS
    except ImportError:
        return
    if not MARGINS:
        return
    tr = terminalreporter
    tr.write_sep("-", "parity margins: case, max-abs error, error/tolerance, ambiguous/rows")
    for case, err, tol, amb, rows in MARGINS:
        tr.write_line(f"{case}: {err:.3e}  {err / tol:.3f}  {amb}/{rows}")
    worst = max(MARGINS, key=lambda m: m[1] / m[2])
    tr.write_line(f"worst: {worst[0]} at {worst[1] / worst[2]:.3f} of its tolerance")
