import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size case, minutes of CPU oracle time")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(autouse=True)
def _no_device_errors(request):
    """After every GPU test: the library's device error word must be clear
    (no bounded wait gave up, no index check failed)."""
    yield
    if "gpu" not in request.keywords:
        return
    import ctypes
    from predictor_gated_channel_b200 import _capi
    bits = ctypes.c_uint(0)
    assert _capi.lib().sfn_device_errors(ctypes.byref(bits), 1) == _capi.SFN_OK
    assert bits.value == 0, f"device error word {bits.value:#x}"
