"""Shared pytest set-up: markers, the CPU oracle, and the independent dense reference."""
import os
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size parity case (minutes)")


def pytest_collection_modifyitems(config, items):
    if torch.cuda.is_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(scope="session")
def oracle():
    import oracle as _oracle
    _oracle.build()
    return _oracle


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Print how many units of each GPU selection swapped a tied page with the oracle's."""
    try:
        from parity import REPORTS
    except Exception:
        return
    if REPORTS:
        terminalreporter.section("selection swaps against the oracle (tie rule)")
        for line in REPORTS:
            terminalreporter.write_line(line)
