import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (sm_100a) and the built library")
    config.addinivalue_line("markers", "slow: long-running CPU check")


def pytest_collection_modifyitems(config, items):
    """Without a GPU, gpu-marked tests are skipped instead of erroring."""
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def pytest_terminal_summary(terminalreporter):
    """Near-tie counts of the GPU parity comparisons (recorded by tests/_parity.py)."""
    try:
        from tests import _parity
    except Exception:  # pragma: no cover
        return
    if not _parity.NEAR_LOG:
        return
    tr = terminalreporter
    tr.write_sep("-", "near-ties (T=0 rows with fp64 top1-top2 < 1e-3; excused = replayed near-ties)")
    tot = dict(requests=0, rows=0, near_rows=0, excused=0)
    for e in _parity.NEAR_LOG:
        tr.write_line(f"{e['test']:<40} requests {e['requests']:>5}  rows {e['rows']:>6}  "
                      f"near {e['near_rows']:>4}  excused {e['excused']:>3}")
        for k in tot:
            tot[k] += e[k]
    tr.write_line(f"{'total':<40} requests {tot['requests']:>5}  rows {tot['rows']:>6}  "
                  f"near {tot['near_rows']:>4}  excused {tot['excused']:>3}")
