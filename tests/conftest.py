import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 GPU and the built CUDA library")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.build()
    return oracle


def pytest_terminal_summary(terminalreporter):
    """Near-threshold decisions of the GPU parity cases: draws whose uniform
    lies within 1e-6 of a decision threshold (or greedy near-ties) are counted
    by the oracle and excluded from the bit-exact comparison."""
    try:
        from parity import NEAR_THRESHOLD
    except ImportError:
        return
    if not NEAR_THRESHOLD:
        return
    tr = terminalreporter
    tr.write_sep("-", "near-threshold rows per parity case (counted, not compared)")
    total_rows = total_flag = 0
    for case, cyc, rows, flagged in NEAR_THRESHOLD:
        tr.write_line(f"{case:40s} cycle {cyc:3d}: {flagged:4d} of {rows:7d} rows")
        total_rows += rows
        total_flag += flagged
    tr.write_line(f"{'total':40s}          : {total_flag:4d} of {total_rows:7d} rows")
