import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size workload (minutes)")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Near-tie report: how many rows of each GPU-vs-oracle selection differ,
    all of them only at blocks whose oracle score lies within 1e-4 of the
    selection threshold (the tolerance of the parity contract)."""
    from tests.parity_utils import ATTN_LOG, TIE_LOG, TIE_TOL
    tr = terminalreporter
    if ATTN_LOG:
        tr.write_sep("-", "attention rows against the oracle (worst max-abs / mean-abs)")
        for label, n, mx, mean in ATTN_LOG:
            tr.write_line(f"{label}: {n} query blocks, {mx:.2e} / {mean:.2e}")
    if not TIE_LOG:
        return
    tr.write_sep("-", f"selection near-ties (score gap < {TIE_TOL:g} to the threshold)")
    total = rows = 0
    for label, ties, n in TIE_LOG:
        tr.write_line(f"{label}: {ties} of {n} rows differ only at near-ties")
        total += ties
        rows += n
    tr.write_line(f"all selections: {total} near-tie rows of {rows} compared")
