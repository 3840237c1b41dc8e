import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size workloads (minutes)")


@pytest.fixture(scope="session")
def orc():
    import oracle

    oracle.build()
    return oracle


def pytest_terminal_summary(terminalreporter):
    # decision-parity and output figures recorded by the GPU parity tests
    parity = sys.modules.get("tests.parity")
    if parity is not None and parity.REPORT:
        terminalreporter.write_line("")
        for line in parity.format_report(parity.REPORT).splitlines():
            terminalreporter.write_line(line)
        # optional machine-readable copy (MALA_PARITY_REPORT=<path.json>)
        path = os.environ.get("MALA_PARITY_REPORT")
        if path:
            import json

            with open(path, "w") as f:
                json.dump(parity.REPORT, f, indent=1)
