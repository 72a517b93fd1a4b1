import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA GPU in this process")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(autouse=True)
def _chunkwise_schedule_for_gpu_tests(request):
    """GPU tests run the chunkwise prefill kernels they were written for: the library's
    automatic schedule would send their small shapes to the column scan, which
    tests/test_scan_gpu.py covers on its own (it sets the schedule it tests)."""
    if request.node.get_closest_marker("gpu") is None:
        yield
        return
    import gated_delta_rule_122_b200 as kda
    prev = kda.get_schedule()
    kda.set_schedule("chunked")
    try:
        yield
    finally:
        kda.set_schedule(prev)
