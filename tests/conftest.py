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
