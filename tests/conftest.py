import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_collection_modifyitems(config, items):
    import torch
    if torch.cuda.is_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """The parity tests' measured errors against the fp64 oracle, per case and
    output tensor: max |x - ref| / max |ref| (the pass metric) and the largest
    elementwise |x - ref| / (|ref| + 1e-3 max |ref|) (for information)."""
    try:
        from tests.helpers import PARITY_REPORT
    except ImportError:
        return
    if not PARITY_REPORT:
        return
    tr = terminalreporter
    tr.write_sep("-", "parity against the fp64 oracle")
    tr.write_line(f"{'case':58s} {'tensor':12s} {'max|d|/max|ref|':>16s} {'elementwise':>12s}")
    for case, tensor, rel, elem in PARITY_REPORT:
        tr.write_line(f"{case[:58]:58s} {tensor:12s} {rel:16.3e} {elem:12.3e}")
