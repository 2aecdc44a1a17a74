import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_terminal_summary(terminalreporter):
    try:
        from _helpers import PARITY_LOG
    except Exception:
        return
    if not PARITY_LOG:
        return
    tr = terminalreporter
    tr.write_sep("-", "parity margins: max|d| / max|oracle| (y, final states) against the tolerance")
    for name, ey, ef, tol in PARITY_LOG:
        fs = "-" if ef is None else f"{ef:.3e}"
        tr.write_line(f"{name:70s} y {ey:.3e}  final {fs:>9s}  tol {tol:.0e}")
