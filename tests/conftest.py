import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
TESTS = os.path.dirname(os.path.abspath(__file__))
if TESTS not in sys.path:
    sys.path.insert(0, TESTS)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Print the layer errors the parity tests recorded (for information: the bars are
    the normwise tolerances asserted in the tests)."""
    try:
        from helpers import ERROR_REPORT
    except ImportError:
        return
    if not ERROR_REPORT:
        return
    tr = terminalreporter
    tr.section("layer errors against the oracle (normwise max rel / per-element)")
    for name, nw, pe in ERROR_REPORT:
        tr.write_line(f"{name:70s} {nw:.3e}  {pe:.3e}")
