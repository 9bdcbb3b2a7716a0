import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: long CPU test (large oracle sample)")


def pytest_terminal_summary(terminalreporter):
    """Near-threshold counts of every GPU mask comparison of the session (the
    mask tolerance: blocks whose oracle score lies within 1e-3 relative of the
    threshold are excused from bit-exactness, counted and reported here)."""
    helpers = sys.modules.get("gpu_helpers")
    tr = terminalreporter
    outs = getattr(helpers, "OUT_STATS", None)
    if outs:
        tr.section("output parity: errors against the oracle on the same kept lists")
        for label, mx, mn in outs:
            tr.write_line(f"{label.split('::')[-1]}: max-abs {mx:.2e} mean-abs {mn:.2e}")
    stats = getattr(helpers, "MASK_STATS", None)
    if not stats:
        return
    tr.section("mask parity: near-threshold blocks")
    tot = {"near": 0, "excused": 0, "outside": 0, "compared": 0}
    for label, r in stats:
        tr.write_line(f"{label.split('::')[-1]}: near {r['near']} excused {r['excused']} "
                      f"outside {r['outside']} compared {r['compared']}")
        for key in tot:
            tot[key] += r[key]
    tr.write_line(f"total: near {tot['near']} excused {tot['excused']} outside {tot['outside']} "
                  f"compared {tot['compared']}")
