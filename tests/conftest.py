import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def orc():
    import oracle

    oracle.build()
    return oracle


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Raw attention error statistics (max-abs, max-rel over |ref| >= 0.1) of the
    comparisons this session ran; also written as JSON to $TV_ERROR_REPORT."""
    from helpers import ERR_STATS

    if not ERR_STATS:
        return
    tr = terminalreporter
    tr.write_sep("-", "attention error vs oracle (max abs | max rel, |ref| >= 0.1 | elements)")
    for k in sorted(ERR_STATS):
        v = ERR_STATS[k]
        tr.write_line(f"{k:60s} {v['max_abs']:.3e} | {v['max_rel_ref_ge_0.1']:.3e} | {v['elements']}")
    path = os.environ.get("TV_ERROR_REPORT")
    if path:
        import json

        with open(path, "w") as f:
            json.dump(ERR_STATS, f, indent=1, sort_keys=True)
