import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    # Without a CUDA device, GPU tests are skipped rather than failed.
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_sessionfinish(session, exitstatus):
    # the parity statistics the GPU tests collected (harness.record), when asked for
    path = os.environ.get("ZERO_PARITY_REPORT")
    if not path:
        return
    harness = sys.modules.get("harness")
    if harness is None or not harness.REPORT:
        return
    import json
    with open(path, "w") as f:
        json.dump(harness.REPORT, f, indent=1, sort_keys=True)
