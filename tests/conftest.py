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


_PARITY_REPORT = []


@pytest.fixture(scope="session")
def parity_report():
    """Tests append (workload, what, max_abs, rel_fro); the terminal summary
    prints them, so the figures appear in a quiet run's output too."""
    return _PARITY_REPORT


def pytest_terminal_summary(terminalreporter):
    if _PARITY_REPORT:
        terminalreporter.write_sep("-", "full-size parity against the oracle")
        for name, what, max_abs, rel in _PARITY_REPORT:
            terminalreporter.write_line(f"{name}: {what}: max_abs {max_abs:.3e} rel_fro {rel:.3e}")
