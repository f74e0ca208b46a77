import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds")


def pytest_terminal_summary(terminalreporter):
    """The near-boundary count of every sampling comparison with the oracle: sequences whose
    uniform lay within 1e-6 of an accept or CDF boundary in the oracle's float64 arithmetic,
    and how many of those the GPU decided differently (allowed only there)."""
    helpers = sys.modules.get("gpu_helpers")
    log = getattr(helpers, "NEAR_LOG", None)
    if not log:
        return
    tr = terminalreporter
    tr.write_sep("-", "near-boundary cases (|u - boundary| < 1e-6) per sampling comparison")
    tr.write_line(f"{'comparison':<56} {'sequences':>10} {'near':>6} {'differ':>7}")
    tot = [0, 0, 0]
    for label, n, flagged, differ in log:
        tr.write_line(f"{label[:56]:<56} {n:>10} {flagged:>6} {differ:>7}")
        tot = [tot[0] + n, tot[1] + flagged, tot[2] + differ]
    tr.write_line(f"{'total':<56} {tot[0]:>10} {tot[1]:>6} {tot[2]:>7}")
