import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


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
def _canary_fill(request):
    """GPU tests run with every output and workspace the binding allocates filled with
    0xFF bytes first (NaN in floats, -1 in integers), so that a kernel which leaves part
    of its output unwritten or reads scratch it never wrote fails the comparison."""
    if "gpu" not in request.keywords:
        yield
        return
    from linear_attention_paged_b200 import build
    build.build()
    from linear_attention_paged_b200 import wa
    old = wa.CANARY
    wa.CANARY = 0xFF
    try:
        yield
    finally:
        wa.CANARY = old
