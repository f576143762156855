import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a) and the built libstar.so")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_terminal_summary(terminalreporter):
    """Per test: how many compared output elements needed the |O| >= 4 allowance of
    tests/harness.py (half a bf16 spacing + 4e-3 instead of 1.5e-2)."""
    h = sys.modules.get("tests.harness")
    if h is None or not h.ALLOWANCE:
        return
    per: dict[str, list[int]] = {}
    for test, _what, relaxed, total in h.ALLOWANCE:
        acc = per.setdefault(test, [0, 0])
        acc[0] += relaxed
        acc[1] += total
    terminalreporter.write_sep("-", "outputs admitted by the |O| >= 4 allowance (per test)")
    for test, (relaxed, total) in per.items():
        terminalreporter.write_line(f"{test}: {relaxed} of {total} elements")
