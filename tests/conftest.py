import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_collection_modifyitems(config, items):
    # GPU tests fail loudly (not skip) when no GPU is present, so a CPU run
    # must deselect them with -m "not gpu".
    pass


def pytest_terminal_summary(terminalreporter):
    """Prints the parity errors the GPU tests measured (tests/parity.py RECORDS)."""
    from tests import parity
    if not parity.RECORDS:
        return
    tr = terminalreporter
    tr.section("measured parity errors")
    for r in parity.RECORDS:
        rest = " ".join(f"{k}={v}" for k, v in r.items() if k not in ("test", "level"))
        tr.write_line(f"{r['test']} [{r['level']}] {rest}")
    parity.dump_records()
