import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA B200 (sm_100a) device")
    config.addinivalue_line("markers", "slow: large oracle work (full-size workloads)")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


@pytest.fixture(autouse=True, scope="session")
def _short_device_wait_cap(request):
    """GPU tests run with a shorter cap on bounded device waits (2^20 polls), so
    that a kernel bug shows up as a prompt ULY_ERR_TIMEOUT instead of a long
    stall; legitimate waits are microseconds."""
    try:
        import torch
        if not torch.cuda.is_available():
            yield
            return
        import ulysses_sequence_parallelism_b200 as U
        U.ulysses_set_wait_limit(1 << 20)
    except Exception:
        yield
        return
    yield
    U.ulysses_set_wait_limit(0)
