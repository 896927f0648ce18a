import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    # A `-m gpu` run on a machine without a GPU should fail loudly, not skip:
    # the parity tests are the point of those runs.  Without `-m gpu`, GPU
    # tests that got selected anyway are skipped when no GPU is present.
    import torch
    if torch.cuda.is_available():
        return
    markexpr = config.getoption("-m") or ""
    if markexpr.strip() == "gpu":
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    # measured error of every parity check that ran (GPU runs): case, max-abs, rel-L2
    try:
        from parity import PARITY_LOG
    except Exception:
        return
    if not PARITY_LOG:
        return
    tr = terminalreporter
    tr.write_sep("-", "parity against the float64 oracle (bound: |d| <= max(1e-2, 2^-8 |ref|) "
                      "per element, rel-L2 5e-3)")
    for case, max_abs, rel in PARITY_LOG:
        tr.write_line(f"{case:<72s} max-abs {max_abs:.3e}  rel-L2 {rel:.3e}")
