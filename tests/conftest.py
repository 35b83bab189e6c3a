import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_collection_modifyitems(config, items):
    # GPU tests are skipped (not failed) where no device exists; the product path
    # itself never falls back to the CPU.
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
    # ZB_PARITY_REPORT=<path>: write every float parity check of the session (per-head
    # error against its bar, and the per-element figure with a floor of 1e-3 max|ref|)
    path = os.environ.get("ZB_PARITY_REPORT")
    if not path:
        return
    try:
        from tests.gpu_helpers import REPORT
    except Exception:  # pragma: no cover
        return
    import json
    os.makedirs(os.path.dirname(os.path.abspath(path)), exist_ok=True)
    with open(path, "w") as f:
        json.dump({"checks": REPORT,
                   "max_per_head": max((r["per_head"] for r in REPORT), default=None),
                   "max_per_element": max((r["per_element"] for r in REPORT), default=None)}, f, indent=1)
