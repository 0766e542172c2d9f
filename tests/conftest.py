import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a) and the built libmsa.so")


def pytest_collection_modifyitems(config, items):
    import torch

    if torch.cuda.is_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device in this process")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


@pytest.fixture(autouse=True)
def _name_parity_comparisons(request):
    """Labels the selection comparisons a test makes with its id (near-tie report)."""
    import parity

    parity.CURRENT_TEST = request.node.nodeid
    yield


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Near-tie rows (cutoff margin < 1e-4, excluded from the bit-exact selection check) per test."""
    try:
        import parity
    except ImportError:
        return
    tr = terminalreporter
    if parity.REPORT_LOG:
        tr.write_sep("-", "achieved errors against the oracle")
        for name, line in parity.REPORT_LOG:
            tr.write_line(f"{name.split('::', 1)[-1]}: {line}")
    if not parity.NEAR_TIE_LOG:
        return
    per = {}
    for name, rows, near, flipped in parity.NEAR_TIE_LOG:
        r = per.setdefault(name, [0, 0, 0])
        r[0] += rows
        r[1] += near
        r[2] += flipped
    tr.write_sep("-", "selection near-ties (margin < 1e-4, excluded from the bit-exact check)")
    tot = [0, 0, 0]
    for name, (rows, near, flipped) in per.items():
        tr.write_line(f"{name.split('::', 1)[-1]}: {near} of {rows} (row, group) pairs near-tied, "
                      f"{flipped} of them selected differently")
        tot = [a + b for a, b in zip(tot, (rows, near, flipped))]
    tr.write_line(f"total: {tot[1]} near-tied of {tot[0]} compared, {tot[2]} selected differently")
