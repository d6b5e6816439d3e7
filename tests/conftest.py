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


def pytest_terminal_summary(terminalreporter):
    """Largest parity errors of the session (per-slice max-norm and elementwise relative)."""
    try:
        from tests.parity import REPORT
    except Exception:
        return
    if not REPORT:
        return
    terminalreporter.write_sep("-", "largest parity errors against the oracle")
    for (dtype, name), v in sorted(REPORT.items()):
        terminalreporter.write_line(f"{dtype:>10}  {name:<22} {v:.3e}")
