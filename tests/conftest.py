import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    # The layer library is built in-tree and not committed: build it once if a
    # fresh checkout does not have it yet (nvcc cross-compiles without a GPU).
    if not os.path.exists(os.path.join(ROOT, "int4_routed_expert_bias_b200", "libcoli.so")):
        import __graft_entry__
        __graft_entry__.build()


def cuda_available():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def pytest_collection_modifyitems(config, items):
    if cuda_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)
