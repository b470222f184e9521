import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


@pytest.fixture(autouse=True)
def _no_device_error_after_gpu_test(request):
    """Every GPU test ends with the library's device error word clear: a
    kernel that recorded an error (an expired wait, or an out-of-range index
    in the index-checking build) fails the test that launched it."""
    yield
    if "gpu" not in request.keywords:
        return
    import bit_jl_key_b200 as jl
    if jl._lib is not None:
        assert jl.jl_device_error() == 0, "device error word set after the test"
