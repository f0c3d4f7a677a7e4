import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the CUDA library")


def pytest_terminal_summary(terminalreporter):
    """Print the errors that parity checks asked to have reported (whole
    workload tensors against the oracle)."""
    parity = sys.modules.get("parity")
    records = getattr(parity, "RECORDS", None)
    if records:
        terminalreporter.write_sep("-", "errors against the fp64 oracle")
        for line in records:
            terminalreporter.write_line(line)
