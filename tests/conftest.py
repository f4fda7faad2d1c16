import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workloads")
    config.addinivalue_line("markers", "unverified: GPU tests of kernels that have not yet run on a B200; "
                                       "not selected by -m gpu, run with -m unverified")


def _cuda_available() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


# Tests of the rows built on top of the core path (backward at full size, SIP, SQuad) run after
# every test of the core path, so that a run stopping at the first failure (-x) never leaves a
# core result unreported because of them.
EXTENSION_MODULES = ("test_gpu_sip", "test_gpu_squad", "test_gpu_wan_backward")


def pytest_collection_modifyitems(config, items):
    def is_extension(item):
        return item.module.__name__.rsplit(".", 1)[-1] in EXTENSION_MODULES

    items[:] = [i for i in items if not is_extension(i)] + [i for i in items if is_extension(i)]
    if _cuda_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords or "unverified" in item.keywords:
            item.add_marker(skip)
