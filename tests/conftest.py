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
def golden_dir():
    return os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def pytest_terminal_summary(terminalreporter):
    """Worst achieved parity error per test (the margins behind the asserts)."""
    import json

    from helpers import MEASURED
    if not MEASURED:
        return
    worst = {}
    for m in MEASURED:
        key = (m["test"], m["what"])
        if key not in worst or m["err"] > worst[key]["err"]:
            worst[key] = m
    tr = terminalreporter
    tr.section("parity margins (worst achieved error per test)")
    for (test, what), m in sorted(worst.items()):
        tr.write_line(f"{m['err']:.3e}  {what:<12} {test}  ({m['where']})")
    path = os.environ.get("RETNET_PARITY_LOG")
    if path:
        os.makedirs(os.path.dirname(os.path.abspath(path)), exist_ok=True)
        with open(path, "w") as f:
            json.dump(MEASURED, f, indent=0)
