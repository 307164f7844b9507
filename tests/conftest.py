import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def read_golden(name):
    """Parse a golden fixture: '<hex code> <value>' lines, '#' comments."""
    out = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            c, v = line.split()
            out.append((int(c, 16), float(v)))
    return out


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Print every parity bar checked in this run with the margin left
    (measured / bar; 1.0 would be at the bar)."""
    parity = sys.modules.get("parity")
    if parity is None:
        return
    rows = parity.MARGINS
    if not rows:
        return
    tr = terminalreporter
    tr.section("parity margins (measured / bar)")
    worst = {}
    for label, what, v, bar in rows:
        r = v / bar if bar > 0 else 0.0
        if what not in worst or r > worst[what][0]:
            worst[what] = (r, label, v, bar)
    for label, what, v, bar in rows:
        tr.write_line(f"{label:48s} {what:22s} {v:10.3e} / {bar:8.1e} = {v / bar if bar else 0:6.3f}")
    tr.write_line("worst per bar:")
    for what, (r, label, v, bar) in sorted(worst.items()):
        tr.write_line(f"  {what:22s} {r:6.3f}  ({label})")
