import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def cuda_ok():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return True


def pytest_terminal_summary(terminalreporter):
    """The parity margins: for each compared tensor, the worst measured error
    of the session against the tolerance of its dtype."""
    try:
        from tests.helpers import margin_report
    except Exception:       # the helpers failed to import: their tests report it
        return
    lines = margin_report()
    if lines:
        terminalreporter.write_sep("-", "parity margins (worst error per tensor / tolerance)")
        for line in lines:
            terminalreporter.write_line(line)
