import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
TESTS = os.path.dirname(os.path.abspath(__file__))
if TESTS not in sys.path:
    sys.path.insert(0, TESTS)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a) and the built library")
    config.addinivalue_line("markers", "slow: long-running GPU parity case")


def pytest_collection_modifyitems(config, items):
    import torch
    if torch.cuda.is_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Print every recorded parity comparison (tests/helpers.check_parity) as one table, and
    write it as JSON lines when KDA_PARITY_LOG names a file."""
    from helpers import PARITY_LOG
    if not PARITY_LOG:
        return
    tr = terminalreporter
    tr.write_sep("-", "parity errors (max rel = max|x-ref|/max|ref|; elem: floor 1% of max|ref|)")
    tr.write_line(f"{'case':44s} {'tensor':8s} {'tol':>7s} {'max rel':>10s} {'worst head':>10s} "
                  f"{'elem':>10s} {'max abs':>10s}")
    for r in PARITY_LOG:
        tr.write_line(f"{r['case'][:44]:44s} {r['tensor'][:8]:8s} {r['tol']:7.0e} {r['rel']:10.3e} "
                      f"{r['head_rel']:10.3e} {r['elem']:10.3e} {r['abs']:10.3e}")
    path = os.environ.get("KDA_PARITY_LOG")
    if path:
        import json
        with open(path, "w") as f:
            for r in PARITY_LOG:
                f.write(json.dumps(r) + "\n")
