import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running")


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


@pytest.fixture(autouse=True, scope="session")
def _short_device_waits():
    """Bounded device waits give up after 0.5 s in tests (default 2 s)."""
    try:
        import torch
        if torch.cuda.is_available():
            from bit_attention_video_02_b200 import build, vca
            build.build()
            vca.set_wait_limit_ns(500_000_000)
    except Exception:  # pragma: no cover - the GPU tests report the failure
        pass
    yield
