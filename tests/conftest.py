import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """One JSON line per GPU parity test with its counts (near-threshold selection
    differences, degenerate pairs and boundary cases, compared rows, worst errors),
    printed after the results so that it survives `-q`."""
    parity = sys.modules.get("parity")
    reports = getattr(parity, "REPORTS", None) if parity else None
    if not reports:
        return
    terminalreporter.write_sep("-", "parity counts (GPU vs oracle, identical inputs each round)")
    for line in reports:
        terminalreporter.write_line("PARITY " + json.dumps(line, sort_keys=True))
