import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config._qsa_notes = []


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Print what the parity tests measured about themselves (rows checked, wall time, cores)."""
    notes = getattr(config, "_qsa_notes", [])
    if notes:
        terminalreporter.section("QSA parity notes")
        for n in notes:
            terminalreporter.write_line(n)


@pytest.fixture(scope="session")
def oracle_lib():
    from oracle import oracle
    oracle.lib()
    return oracle
