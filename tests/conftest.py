import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a)")


def pytest_collection_modifyitems(config, items):
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


@pytest.fixture(autouse=True)
def _fresh_device_status(request):
    """The library's device status word is sticky (the first error wins), so
    every GPU test starts from a cleared word: one failing test must not
    fail the ones after it."""
    if "gpu" in request.keywords:
        import torch
        import trainable_block_sparse_pool_b200 as T
        torch.cuda.synchronize()
        T.infllm2_clear_device_status()
    yield
