import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_collection_modifyitems(config, items):
    import torch
    if torch.cuda.is_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(autouse=True)
def _no_index_check_fired(request):
    """With the checks build loaded (GDR_LIBRARY=checks), every GPU test must leave the
    device-side index-check word clear."""
    yield
    if os.environ.get("GDR_LIBRARY") != "checks" or "gpu" not in request.keywords:
        return
    import torch
    if not torch.cuda.is_available():
        return
    import gated_delta_rule_79_b200 as g
    g.check_status()
