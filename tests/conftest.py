import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running case")


@pytest.fixture(scope="session")
def cuda_ok():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return True


def pytest_terminal_summary(terminalreporter):
    """Print the parity errors (normwise bound and elementwise figure) of
    every GPU-vs-oracle comparison this run made."""
    try:
        from tests import parity
    except Exception:
        return
    if not parity.REPORT:
        return
    tr = terminalreporter
    tr.write_sep("-", "parity: normwise (bounded) | elementwise, floor 1e-3 max|ref| (reported)")
    for what, norm, elem in parity.REPORT:
        tr.write_line("%-44s out %.2e M %.2e z %.2e | out %.2e M %.2e z %.2e" % ((what[:44],) + norm + elem))
