import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    import torch
    if torch.cuda.is_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


@pytest.fixture(autouse=True)
def _no_bounds_violation(request):
    """With the bounds-checked library loaded (GQ4_LIBRARY pointing at
    libgq4_checked.so), every GPU test must leave the bounds status word clear: valid
    inputs never produce an index outside its array."""
    yield
    if "gpu" not in request.keywords:
        return
    import torch
    if not torch.cuda.is_available():
        return
    from weight_only_int4_gq4_b200 import gq4
    if gq4.build_checked():
        assert gq4.bounds_status(clear=True) == 0, "an index fell outside its array"
