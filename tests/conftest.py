import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU")
    config.addinivalue_line("markers", "slow: long CPU test")


def read_golden(name):
    """Non-comment lines of a golden fixture, split into tokens."""
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# Parity margins seen by the GPU tests: per test, the largest max|gpu - ref| /
# max|ref| over the tensors it compared and the near-tie argmax count, printed
# at the end of the session so that a drift toward the tolerance shows.
MARGINS = {}


def record_margin(err=None, near_tie=False, route_tie=False):
    test = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
    m = MARGINS.setdefault(test, {"max_rel_err": 0.0, "compared": 0, "near_ties": 0, "route_ties": 0})
    if err is not None:
        m["max_rel_err"] = max(m["max_rel_err"], float(err))
        m["compared"] += 1
    if near_tie:
        m["near_ties"] += 1
    if route_tie:
        m["route_ties"] += 1


def pytest_terminal_summary(terminalreporter):
    if not MARGINS:
        return
    terminalreporter.write_line("parity margins (max |gpu - ref| / max |ref| per test; tolerance 2e-2):")
    for test, m in sorted(MARGINS.items()):
        terminalreporter.write_line(f"  {m['max_rel_err']:.3e}  over {m['compared']:4d} tensors, "
                                    f"{m['near_ties']} near-tie argmax, {m['route_ties']} near-tie routings  {test}")
