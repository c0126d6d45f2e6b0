import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter):
    """Measured error of every GPU-vs-oracle comparison of the session, as a
    fraction of its bar (1.0 = at the bar), so each run's log shows the
    margins and not only pass or fail."""
    try:
        from gpu_helpers import BF16_TOL, F32_TOL, RECORDED
    except Exception:
        return
    if not RECORDED:
        return
    tr = terminalreporter
    tr.write_sep("-", "measured error / bar per comparison")
    for label, dtype, errs in RECORDED:
        bar = F32_TOL if dtype == "f32" else BF16_TOL
        cells = " ".join("%s=%.3f" % (n, e / bar) for n, e in errs.items())
        tr.write_line("%-60s %s" % (label[:60], cells))
