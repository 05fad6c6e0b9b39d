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
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload, minutes of host work")


def pytest_terminal_summary(terminalreporter):
    """Print the worst error / bound of every GPU-vs-oracle comparison (1.0
    is the tolerance), largest first, with the number of elements compared."""
    try:
        import gpu_util
    except Exception:
        return
    if not gpu_util.MARGINS:
        return
    rows = sorted(gpu_util.MARGINS, key=lambda r: -r[3])
    tr = terminalreporter
    tr.section("parity margins (worst error / bound; 1.0 = tolerance)")
    worst = {}
    for test, name, n, m in rows:
        key = (test, name)
        if key not in worst or m > worst[key][1]:
            worst[key] = (n, m)
    ranked = sorted(worst.items(), key=lambda kv: -kv[1][1])
    for (test, name), (n, m) in ranked[:80]:
        tr.write_line(f"{m:8.4f}  {n:>11d}  {name:<14s} {test}")
    if len(ranked) > 80:
        tr.write_line(f"... {len(ranked) - 80} more comparisons, all below {ranked[80][1][1]:.4f}")
