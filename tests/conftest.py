import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the CUDA library")


def pytest_collection_modifyitems(config, items):
    # GPU tests are skipped (not failed) when no GPU is present and -m gpu was not asked for
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def pytest_sessionfinish(session, exitstatus):
    # the parity comparisons' agreement figures, when asked for (DQ_PARITY_REPORT=<path>)
    path = os.environ.get("DQ_PARITY_REPORT")
    if not path:
        return
    try:
        from tests import _parity
    except Exception:  # pragma: no cover
        return
    import json
    with open(path, "w") as fh:
        json.dump(_parity.REPORTS, fh, indent=1)
