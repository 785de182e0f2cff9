import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def oracle():
    import oracle as _oracle
    _oracle.build()
    return _oracle


def pytest_terminal_summary(terminalreporter):
    """Print the parity errors that tests recorded (record_property), one line per test."""
    rows = []
    for rep in terminalreporter.stats.get("passed", []) + terminalreporter.stats.get("failed", []):
        props = [(k, v) for k, v in getattr(rep, "user_properties", []) if k.endswith("_err")]
        if props and rep.when == "call":
            rows.append((rep.nodeid, props))
    if rows:
        terminalreporter.write_sep("-", "recorded parity errors (max|err| / max|oracle|)")
        for nodeid, props in rows:
            terminalreporter.write_line(nodeid.split("::", 1)[-1] + "  " +
                                        "  ".join(f"{k}={v:.2e}" for k, v in props))
