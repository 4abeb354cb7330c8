import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running")


def pytest_terminal_summary(terminalreporter):
    """Parity diagnostics beside the gates: for every decode comparison with
    the oracle, max|err| against its tolerance, the relative RMS error and
    max|ref| (for the lse rows, max|err| is the absolute log-sum-exp error)."""
    try:
        from tests import helpers
    except Exception:
        return
    if not helpers.DIAG:
        return
    tr = terminalreporter
    tr.section("parity diagnostics (decode vs oracle)")
    tr.write_line("%-58s %11s %11s %10s %10s" % ("case", "max|err|", "tol", "rel-RMS", "max|ref|"))
    for what, err, t, rr, mx in helpers.DIAG:
        tr.write_line("%-58s %11.3e %11.3e %10.2e %10.3e" % (what[:58], err, t, rr, mx))
    lse = [x for x in helpers.DIAG if x[0].endswith(" lse")]
    out = [x for x in helpers.DIAG if x[0].endswith(" out")]
    if out:
        tr.write_line("worst out rel-RMS %.2e; worst out max|err|/tol %.3f" % (
            max(x[3] for x in out), max(x[1] / x[2] for x in out if x[2] > 0)))
    if lse:
        tr.write_line("worst |d lse| %.3e; worst lse max|err|/tol %.3f" % (
            max(x[1] for x in lse), max(x[1] / x[2] for x in lse if x[2] > 0)))
