import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: large sizes")


def pytest_terminal_summary(terminalreporter):
    """Totals of the selection decisions the parity tests checked: exact (the
    GPU list equals the oracle's) and near-tied (band rules only)."""
    exact = near = 0
    for name in ("tests.pair", "pair"):
        mod = sys.modules.get(name)
        if mod is not None:
            exact += mod.SELECTION_STATS["exact"]
            near += mod.SELECTION_STATS["near_tie"]
    if exact or near:
        terminalreporter.write_line(
            f"selection decisions checked: {exact} exact, {near} near-tied (band rules)")
