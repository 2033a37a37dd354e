import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running (full-size workloads)")


def pytest_collection_modifyitems(config, items):
    # GPU tests are skipped only when no CUDA device exists at all; on a GPU
    # machine a missing or broken extension fails loudly instead.
    try:
        import torch
        have_cuda = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_cuda = False
    if have_cuda:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(scope="session", autouse=True)
def _parity_report():
    """With PA_PARITY_REPORT=<path>, write every GPU-vs-oracle comparison of
    the session (name, max-abs, mean-abs, relative L2, LSE relative error) to
    that JSON file at the end."""
    yield
    path = os.environ.get("PA_PARITY_REPORT")
    if path:
        from tests import _parity
        with open(path, "w") as f:
            json.dump(_parity.RECORDED, f, indent=1)
