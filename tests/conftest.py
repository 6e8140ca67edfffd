import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100) GPU and the built libmoeq.so")
    config.addinivalue_line("markers", "slow: long CPU-only check, skipped unless MOEQ_SLOW=1")


def pytest_collection_modifyitems(config, items):
    import torch
    have_gpu = torch.cuda.is_available()
    slow = os.environ.get("MOEQ_SLOW") == "1"
    for it in items:
        if "gpu" in it.keywords and not have_gpu:
            it.add_marker(pytest.mark.skip(reason="no CUDA device"))
        if "slow" in it.keywords and not slow:
            it.add_marker(pytest.mark.skip(reason="set MOEQ_SLOW=1"))
