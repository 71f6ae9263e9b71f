"""NEXT-4: the QKV and output projections with the all-to-alls folded into the
GEMMs, against the fp64 oracle: the QKV GEMM's head-shard outputs equal the
oracle's projection followed by its seq->head all-to-all, the output GEMM
reading head shards equals the oracle's head->seq all-to-all followed by its
projection, and the projected forward block matches the oracle chain."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_util import f64, assert_close

pytestmark = pytest.mark.gpu


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


SHAPES = [
    # N,    P, H, H_kv, d,  hidden
    (1024, 2, 8, 2, 128, 1024),
    (1024, 4, 8, 4, 64, 512),
    (384, 1, 4, 4, 64, 256),      # P = 1, three 128-row tiles, one 256-column tile per tensor group
]


@pytest.mark.parametrize("N,P,H,H_kv,d,hidden", SHAPES)
def test_qkv_projection_into_head_shards(N, P, H, H_kv, d, hidden):
    import ulysses_sequence_parallelism_b200 as U
    x, w_qkv, _ = workloads.projection_inputs(N, H, H_kv, d, hidden, seed=N + hidden)
    x_seq = [_dev(s) for s in workloads.seq_shards(x, P)]
    mk = lambda hx: [torch.empty(N, hx // P, d, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    qh, kh, vh = mk(H), mk(H_kv), mk(H_kv)
    U.ulysses_qkv_proj_seq_to_head(x_seq, _dev(w_qkv), qh, kh, vh, N, P, H, H_kv, d, hidden)
    torch.cuda.synchronize()
    assert U.ulysses_get_device_status() == (0, 0)
    w = oracle.widen_bf16
    q_s, k_s, v_s = oracle.qkv_projection(workloads.seq_shards(w(x), P), w(w_qkv), H, H_kv, d)
    for name, got, ref in (("Q", qh, q_s), ("K", kh, k_s), ("V", vh, v_s)):
        refh = oracle.seq_to_head(ref)
        for r in range(P):
            assert_close(f"{name} rank {r}", f64(got[r]), refh[r])


@pytest.mark.parametrize("N,P,H,H_kv,d,hidden", SHAPES)
def test_out_projection_from_head_shards(N, P, H, H_kv, d, hidden):
    import ulysses_sequence_parallelism_b200 as U
    _, _, w_o = workloads.projection_inputs(N, H, H_kv, d, hidden, seed=7)
    rng = np.random.Generator(np.random.PCG64(N + P))
    o = workloads.round_to_bf16_bits(rng.standard_normal((N, H, d), dtype=np.float32))
    o_head = oracle.seq_to_head(workloads.seq_shards(o, P))                   # bit patterns, head layout
    oh = [_dev(t) for t in o_head]
    y = [torch.empty(N // P, hidden, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    U.ulysses_out_proj_head_to_seq(oh, _dev(w_o), y, N, P, H, H_kv, d, hidden)
    torch.cuda.synchronize()
    assert U.ulysses_get_device_status() == (0, 0)
    w = oracle.widen_bf16
    ref = oracle.out_projection(workloads.seq_shards(w(o), P), w(w_o))
    for p in range(P):
        assert_close(f"Y shard {p}", f64(y[p]), ref[p])


def test_projected_forward_block_matches_oracle():
    import ulysses_sequence_parallelism_b200 as U
    N, P, H, H_kv, d, hidden = 1024, 2, 8, 2, 128, 1024
    cu = [0, 300, 301, 1024]
    x, w_qkv, w_o = workloads.projection_inputs(N, H, H_kv, d, hidden, seed=3)
    layer = U.UlyssesLayer(N, P, H, H_kv, d, cu_seqlens=torch.tensor(cu, dtype=torch.int32, device="cuda"),
                           backward=False)
    y = layer.forward_projected([_dev(s) for s in workloads.seq_shards(x, P)], _dev(w_qkv), _dev(w_o))
    torch.cuda.synchronize()
    assert U.ulysses_get_device_status() == (0, 0)
    w = oracle.widen_bf16
    q_s, k_s, v_s = oracle.qkv_projection(workloads.seq_shards(w(x), P), w(w_qkv), H, H_kv, d)
    o_s, _ = oracle.ulysses_layer_forward(q_s, k_s, v_s, cu)
    ref = oracle.out_projection(o_s, w(w_o))
    for p in range(P):
        assert_close(f"Y shard {p}", f64(y[p]), ref[p])
