import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU")


# Lines that tests add to the end-of-run summary (the parity statistics of the
# full-size workloads), printed even in quiet mode.
_SUMMARY = []


@pytest.fixture(scope="session")
def summary_lines():
    return _SUMMARY


def pytest_terminal_summary(terminalreporter):
    if _SUMMARY:
        terminalreporter.write_sep("-", "parity statistics")
        for line in _SUMMARY:
            terminalreporter.write_line(line)


@pytest.fixture(scope="session")
def orc():
    """The C oracle, built if needed."""
    import oracle
    return oracle.load()


def _cuda_ok():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def pytest_collection_modifyitems(config, items):
    if _cuda_ok():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)
