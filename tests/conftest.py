import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def read_golden(name):
    """Non-comment lines of a golden fixture, split into fields."""
    rows = []
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


def pytest_terminal_summary(terminalreporter):
    """Prints the attention error figures the parity tests recorded (shown under -q too)."""
    try:
        from oracle_side import ERRORS
    except ImportError:
        return
    if not ERRORS:
        return
    tr = terminalreporter
    tr.write_sep("-", "attention vs the fp64 oracle: max abs / max rel error (|ref| > 1e-3)")
    for name, n, abs_err, rel_err in ERRORS:
        tr.write_line("%-44s %10d outputs  max abs %.3e  max rel %.3e" % (name, n, abs_err,
                                                                           rel_err))
