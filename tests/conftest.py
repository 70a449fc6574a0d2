import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a B200 (sm_100a) GPU and the built libfa2")
    config.addinivalue_line(
        "markers", "slow: large oracle runs (full-size sampled heads)")


def pytest_collection_modifyitems(config, items):
    # GPU tests need a device; say so plainly instead of failing obscurely.
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device visible")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(autouse=True)
def _device_status_word(request):
    """GPU tests start with a clear device status word and must leave it
    clear: a kernel that gave up a bounded wait is reported against the test
    that launched it, not a later one."""
    if "gpu" not in request.keywords:
        yield
        return
    from exact_attention_147_b200 import fa2 as F
    F.device_status(clear=True)
    yield
    code = F.device_status(clear=True)
    assert code == 0, f"device status {code:#x} left by this test"
