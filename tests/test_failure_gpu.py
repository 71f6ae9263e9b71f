"""Failure detection without a GPU fault: a bounded device wait that runs out
records an error word the host reads back, and the context stays usable."""
import numpy as np
import pytest
import torch

from tests.test_attn_gpu import _draw, run_gpu_layer, oracle_layer, check

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports():
    import ulysses_sequence_parallelism_b200 as U
    assert U.ulysses_get_device_status() == (0, 0)
    U.ulysses_set_wait_limit(1000)
    try:
        U.ulysses_selftest_bounded_wait()
        code, word = U.ulysses_get_device_status()
    finally:
        U.ulysses_set_wait_limit(1 << 20)      # the session's test cap (see conftest)
    assert code == 4                       # ULY_ERR_TIMEOUT
    assert word == (0x7F << 24) | 0xABC    # kernel id, site
    assert U.ulysses_get_device_status() == (0, 0)   # read-and-clear
    # the context is intact: a normal layer step still matches the oracle
    q, k, v, do = _draw(256, 4, 2, 128, seed=23)
    check(run_gpu_layer(q, k, v, do, 2, [0, 77, 256]), oracle_layer(q, k, v, do, 2, [0, 77, 256]))
