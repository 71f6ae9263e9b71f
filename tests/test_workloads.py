"""Host-side checks of the seeded input generators (no GPU)."""
import numpy as np
import torch

import workloads


def test_bf16_rounding_is_round_to_nearest_even():
    rng = np.random.Generator(np.random.PCG64(1))
    x = np.concatenate([rng.standard_normal(100000, dtype=np.float32),
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 0.0, -0.0], np.float32)])
    ours = workloads.round_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_doc_lengths_cover_N_within_bounds():
    rng = np.random.Generator(np.random.PCG64(0))
    L = workloads.draw_doc_lengths(rng, 65536, 1024, 16384)
    assert sum(L) == 65536
    assert all(1 <= x <= 16384 for x in L)
    assert all(x >= 1024 for x in L[:-1])
    cu = workloads.cu_seqlens_from_lengths(L)
    assert cu[0] == 0 and cu[-1] == 65536 and np.all(np.diff(cu) > 0)


def test_generation_is_deterministic_and_shaped():
    w = workloads.get("varlen64k")
    a = workloads.generate(w, N=4096)
    b = workloads.generate(w, N=4096)
    assert np.array_equal(a["q"], b["q"]) and np.array_equal(a["cu_seqlens"], b["cu_seqlens"])
    assert a["q"].shape == (4096, 32, 128) and a["k"].shape == (4096, 8, 128)
    assert a["do"].shape == (4096, 32, 128)


def test_pair_count():
    assert workloads.causal_pairs(512) == 131328
    assert workloads.causal_pairs(8192) == 33558528
    assert workloads.causal_pairs(98304) == 4831887360
    assert workloads.causal_pairs(6, [0, 2, 6]) == 3 + 10
