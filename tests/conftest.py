import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU test collected but no CUDA device is visible")
    return torch.device("cuda:0")


def pytest_terminal_summary(terminalreporter):
    """One line per full-size parity comparison: the observed errors."""
    try:
        from tests.helpers import PARITY_LOG
    except Exception:
        return
    rows = [e for e in PARITY_LOG if e[0].startswith("full ")]
    if not rows:
        return
    terminalreporter.write_line("parity at full size (max-abs, max row-relative error):")
    for what, mx, rel in rows:
        terminalreporter.write_line("  %-28s max-abs %.3e%s" % (
            what, mx, "" if rel is None else "  row-rel %.3e" % rel))
