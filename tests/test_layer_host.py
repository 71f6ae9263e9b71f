"""UlyssesLayer argument checks that run before any device allocation (CPU)."""
import pytest

import ulysses_sequence_parallelism_b200 as U


@pytest.mark.parametrize("kw", [
    dict(head_fragment=3),                           # not a multiple of the GQA group (H/H_kv = 4)
    dict(head_fragment=4, fused=True),               # fragmentation excludes the fused layer
    dict(head_fragment=4, rank_sequential=True),     # and rank-sequential processing
    dict(head_fragment=16),                          # does not divide H/P = 8
])
def test_bad_head_fragment_rejected(kw):
    with pytest.raises(ValueError):
        U.UlyssesLayer(1024, 4, 32, 8, 128, device="cpu", **kw)


def test_fused_needs_shards_of_128_tokens():
    with pytest.raises(ValueError):
        U.UlyssesLayer(1000, 4, 32, 8, 128, device="cpu", fused=True)     # N/P = 250


def test_too_many_ranks_rejected():
    with pytest.raises(ValueError):
        U.UlyssesLayer(4096, 32, 32, 32, 128, device="cpu")
