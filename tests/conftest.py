import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter):
    """Print (and, with DSA_PARITY_STATS=path, save as JSON) how much of each
    parity tolerance the GPU checks used, per workload."""
    from tests import parity_util as pu
    if not pu.STATS:
        return
    terminalreporter.section("parity tolerance use")
    for line in pu.stats_table():
        terminalreporter.write_line(line)
    path = os.environ.get("DSA_PARITY_STATS")
    if path:
        import json
        with open(path, "w") as f:
            json.dump({k: dict(v) for k, v in pu.STATS.items()}, f, indent=1)
