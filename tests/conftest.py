import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds")


def read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line)
    return rows


def page_figures():
    out = {}
    for row in read_golden("page_figures.txt"):
        k, v = (s.strip() for s in row.split("=", 1))
        out[k] = v
    return out


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Print the near-boundary exemption counts the GPU parity tests recorded."""
    gc = sys.modules.get("gpu_common")
    rows = getattr(gc, "PARITY_COUNTS", None) if gc else None
    if not rows:
        return
    tr = terminalreporter
    worst = getattr(gc, "OUT_WORST", None)
    if worst and worst["ratio"] > 0:
        tr.section("attention outputs vs the oracle")
        tr.write_line(f"worst error / bound {worst['ratio']:.3f} (error {worst['err']:.3g} at "
                      f"|o| = {worst['abs_o']:.3g})")
    tr.section("near-boundary exemptions (codes / sign bits inside the 1e-5 band)")
    tot = {}
    for label, counts in rows:
        tr.write_line(f"{label}: " + ", ".join(f"{k}={v}" for k, v in counts.items()))
        for k, v in counts.items():
            tot[k] = tot.get(k, 0) + v
    tr.write_line("total: " + ", ".join(f"{k}={v}" for k, v in tot.items()))
