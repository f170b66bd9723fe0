import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter):
    """Worst per-slice relative L2 error of each recorded parity check, with
    its bar, so the margin shows in the run's output (also under -q)."""
    mod = sys.modules.get("m3_testutil")
    rows = getattr(mod, "MARGINS", None) if mod is not None else None
    if not rows:
        return
    terminalreporter.write_sep("-", "worst per-slice relative L2 error vs the oracle (bar)")
    for name, err, tol in rows:
        terminalreporter.write_line(f"{name}: {err:.3e} ({tol:g}, margin x{tol / max(err, 1e-30):.0f})")
