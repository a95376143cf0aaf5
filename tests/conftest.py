import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# (case, max_abs, rel_l2) of the workload parity checks, printed in the
# terminal summary so a quiet run still shows the measured errors.
_PARITY = []


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA B200 (sm_100a) device")
    config.addinivalue_line("markers", "slow: long-running CPU oracle case")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle

    oracle.build()
    return oracle


@pytest.fixture
def parity_log(record_property):
    def log(case, max_abs, rel_l2):
        _PARITY.append((case, float(max_abs), float(rel_l2)))
        record_property("max_abs", float(max_abs))
        record_property("rel_l2", float(rel_l2))

    return log


def pytest_terminal_summary(terminalreporter):
    if not _PARITY:
        return
    terminalreporter.write_line("")
    terminalreporter.write_line("parity vs oracle (bar: max_abs <= 2e-2, rel_l2 <= 1e-2):")
    for case, ma, rl in _PARITY:
        terminalreporter.write_line(f"  {case}: max_abs={ma:.3e} rel_l2={rl:.3e}")
