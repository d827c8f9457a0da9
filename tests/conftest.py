import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_terminal_summary(terminalreporter):
    """The GPU parity cases' near-tie counts and worst errors, one line each."""
    mod = sys.modules.get("_gpu")
    rep = getattr(mod, "REPORT", None) if mod else None
    if not rep:
        return
    tr = terminalreporter
    tr.write_line("parity report: case decisions near_ties flipped worst_rel_l2(tensor) worst_max_abs")
    for case, r in rep.items():
        tr.write_line(f"  {case} {r['decisions']} {r['near_ties']} {r['flipped']} "
                      f"{r['rel_l2']:.2e}({r['worst']}) {r['max_abs']:.2e}")
