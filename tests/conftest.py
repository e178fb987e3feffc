import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built library")
    config.addinivalue_line("markers", "cpu: CPU-only check")
    config.addinivalue_line("markers", "slow: full-size case, minutes on the CPU oracle")


def read_golden(name):
    """Parse a golden fixture: '#' comments, 'key: values' lines or 'value expected' rows."""
    kv, rows = {}, []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if ":" in line:
                k, v = line.split(":", 1)
                kv[k.strip()] = v.split()
            else:
                rows.append(line.split())
    return kv, rows


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Report how many bf16 rounding flips the output comparisons accepted."""
    try:
        import devutil
    except Exception:
        return
    log = getattr(devutil, "FLIP_LOG", [])
    if not log:
        return
    n = sum(e[1] for e in log)
    flips = sum(e[2] for e in log)
    with_flips = [e for e in log if e[2]]
    worst = max(e[3] for e in log)
    terminalreporter.write_line(
        f"bf16 output comparisons: {len(log)} calls, {n} elements, {flips} rounding flips accepted "
        f"(<= 2 bf16 ulps each) in {len(with_flips)} calls; worst other |err| = {worst:.3e} x RMS")
    for what, size, f, w in sorted(with_flips, key=lambda e: -e[2] / e[1])[:10]:
        terminalreporter.write_line(f"  {what}: {f} of {size} elements")
