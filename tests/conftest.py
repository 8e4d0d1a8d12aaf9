import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(autouse=True)
def _checks_build_guards(request):
    """With MOE_CHECKS=1 (the bounds-checking build of the library): after
    every GPU test, no device bounds check may have failed and every guard
    zone of every live workspace must still hold its canary bytes."""
    yield
    if "gpu" not in request.node.keywords:
        return
    from fine_grained_moe_fp32_b200 import moe as M
    if not M.CHECKS:
        return
    import torch
    torch.cuda.synchronize()
    assert M.device_status() != M.MOE_ERR_BOUNDS, "a device bounds check failed"
    bad = M.check_guards()
    assert not bad, f"guard zones overwritten: {bad[:8]}"
