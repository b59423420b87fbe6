"""Shared test configuration.

Markers:
  gpu  -- needs a CUDA device (sm_100a); parity tests of the CUDA library.
Everything unmarked runs on the CPU in a few minutes.

Parity tests record the error they measured against the tolerance they check
(``record_margin``); the terminal summary lists them, so a run shows how close
each comparison came to its bound even with ``-q``.
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

MARGINS = []


def record_margin(name, quantity, error, tolerance):
    """Remember one measured error next to the tolerance it was checked against."""
    MARGINS.append((name, quantity, float(error), float(tolerance)))


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) CUDA device")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    if not MARGINS:
        return
    tr = terminalreporter
    tr.section("parity margins (measured error / tolerance)")
    worst = max(MARGINS, key=lambda m: m[2] / m[3] if m[3] else 0.0)
    for name, qty, err, tol in MARGINS:
        tr.write_line(f"{name:<58} {qty:<10} {err:.3e} / {tol:.0e}  ({err / tol:6.1%} of bound)")
    tr.write_line(f"largest fraction of its bound: {worst[0]} {worst[1]} {worst[2] / worst[3]:.1%}")
