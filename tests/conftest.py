import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA GPU on this machine")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(autouse=True)
def _short_device_watchdog(request):
    """GPU tests run with a short bounded-wait limit (~67 ms per wait) so that
    a pipeline bug surfaces as MLSTM_ERR_TIMEOUT quickly instead of slowly."""
    if "gpu" not in request.keywords:
        yield
        return
    from mlstm_chunkwise_b200 import api
    api.set_watchdog(1 << 22)
    yield
    api.set_watchdog(0)
