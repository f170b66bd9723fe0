import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


BOUNDS = os.environ.get("M3_BOUNDS", "") == "1"


@pytest.fixture(autouse=True)
def _bounds_build_records(request):
    """Under M3_BOUNDS=1 (the bounds build of the library): after every GPU
    test, any failed device index check of its kernels fails the test."""
    yield
    if BOUNDS and request.node.get_closest_marker("gpu") is not None:
        import state_space_sequence_ssm_b200 as m3
        assert m3.device_checks(), "M3_BOUNDS=1 but the normal build is loaded"
        m3.stream_status()  # raises M3Error(M3_ERR_BOUNDS) with the site, index and extent


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
