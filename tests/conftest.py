import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built libisd.so")
    config.addinivalue_line("markers", "slow: long-running check")


def golden_path(name: str) -> str:
    return os.path.join(ROOT, "tests", "golden", name)


@pytest.fixture
def golden():
    return golden_path


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Accept-parity counts of the GPU tests: requests compared, decisions
    skipped as within 1e-5 of their uniform, inverse-CDF draws whose token
    differs by a rounding-explained neighbouring bucket, and mismatches."""
    mod = sys.modules.get("gpu_util")
    rows = getattr(mod, "PARITY_REPORT", None) if mod else None
    if not rows:
        return
    tr = terminalreporter
    tr.write_line("accept parity (requests / near-threshold / draws / excused draws / mismatches):")
    tot = [0, 0, 0, 0, 0]
    for label, r in rows:
        vals = [r.get("requests", 0), r.get("near_threshold", 0), r.get("draws", 0),
                r.get("excused_draws", 0), r.get("mismatches", 0)]
        tot = [a + b for a, b in zip(tot, vals)]
        tr.write_line("  %-48s %6d %4d %6d %4d %4d" % (label[:48], *vals))
    tr.write_line("  %-48s %6d %4d %6d %4d %4d" % ("total", *tot))
