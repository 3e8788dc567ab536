import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")

HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_terminal_summary(terminalreporter):
    """Per-workload parity table of the full-size tests (shown even with -q)."""
    mod = sys.modules.get("gpu_helpers")
    rows = getattr(mod, "ERROR_REPORT", None) if mod else None
    if not rows:
        return
    tr = terminalreporter
    tr.write_sep("-", "full-size parity against the fp64 oracle")
    tr.write_line(f"{'workload':<24} {'rows':>8} {'max abs err':>12} {'tol':>8} {'lse err':>10}  call")
    for wl, call, n, err, lse_err, tol in rows:
        tr.write_line(f"{wl:<24} {n:>8} {err:>12.3e} {tol:>8.0e} {lse_err:>10.2e}  {call}")
