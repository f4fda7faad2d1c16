import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workloads")


def _cuda_available() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


# Tests of the rows built on top of the core path (backward at full size, SIP, SQuad, fine groups)
# run after every test of the core path, so that a run stopping at the first failure (-x) never
# leaves a core result unreported because of them.  The allocation-free entry point's test runs
# last of all.
EXTENSION_MODULES = ("test_gpu_sip", "test_gpu_squad", "test_gpu_fine", "test_gpu_wan_backward")
LAST_MODULES = ("test_zz_no_alloc",)


def pytest_collection_modifyitems(config, items):
    def rank(item):
        name = item.module.__name__.rsplit(".", 1)[-1]
        return 2 if name in LAST_MODULES else 1 if name in EXTENSION_MODULES else 0

    items[:] = sorted(items, key=rank)          # stable: keeps the collection order within a rank
    if _cuda_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)
