import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Near-cut exemptions of the kept-set comparisons, per workload: they are
    counted, never failed, and reported here at the end of every run."""
    mod = sys.modules.get("tests.parity")
    if mod is None or not mod.REPORT:
        return
    tr = terminalreporter
    tr.write_sep("-", "kept-set exemptions (query blocks checked / near tau / near swap)")
    for label in sorted(mod.REPORT):
        n, tau, swap = mod.REPORT[label]
        tr.write_line(f"{label}: {n} / {tau} / {swap}")


@pytest.fixture(scope="session")
def lib():
    """The C-ABI library (loaded without touching a GPU)."""
    from cross_model_attention_block_b200 import mapflow
    return mapflow.load_library()
