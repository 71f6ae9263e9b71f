"""The multi-process exchange's CUDA pieces on one GPU.

1. ulysses_a2a_pack / ulysses_a2a_unpack, bit for bit: P ranks' packs are run
   one after another on one GPU, the all-to-all between them is done by
   copying chunk q of every rank's send buffer into rank q's receive buffer,
   and each rank's receive buffer must equal the oracle's all-to-all
   restricted to the chunk's heads; unpacking the chunks sent back must
   rebuild exactly the chunk's head columns of every sequence shard and leave
   the other columns untouched.
2. UlyssesDistLayer over a real NCCL process group of one process (P = 1):
   forward and backward against the fp64 oracle, and bit-identical to the
   single-process layer's deterministic kernels.
"""
import os
import socket

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_util import assert_close, bits_of, f64, shards_to_dev, to_dev

pytestmark = pytest.mark.gpu


def _draw(shape, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    return workloads.round_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32))


@pytest.mark.parametrize("N,P,H,H_kv,d,chunk", [
    (512, 2, 8, 4, 64, (0, 4)),        # all heads of a rank in one chunk
    (512, 2, 8, 4, 64, (2, 2)),        # second GQA group only
    (1024, 4, 32, 8, 128, (4, 4)),     # Llama shape, second chunk of two
    (776, 8, 32, 8, 128, (0, 4)),      # one kv head per rank; 97 tokens per rank (ragged)
    (384, 4, 16, 16, 128, (1, 2)),     # MHA, a chunk inside the rank's 4 heads
])
def test_pack_unpack_bit_exact(N, P, H, H_kv, d, chunk):
    import ulysses_sequence_parallelism_b200 as U
    lo, f = chunk
    g = H // H_kv
    n = N // P
    xs = [_draw((N, hx, d), 10 + i) for i, hx in enumerate((H, H_kv, H_kv))]
    seq = [shards_to_dev(x, P) for x in xs]                  # seq[t][p]: rank p's shard of tensor t
    fs = [f, f // g, f // g]
    los = [lo, lo // g, lo // g]
    send = [[torch.full((P, n, fs[t], d), -1.0, dtype=torch.bfloat16, device="cuda") for t in range(3)]
            for _ in range(P)]
    for p in range(P):
        U.ulysses_a2a_pack(seq[0][p], seq[1][p], seq[2][p], *send[p], N, P, H, H_kv, d, lo, f)
    # the all-to-all: rank q receives chunk q of every rank, in source-rank order
    recv = [[torch.stack([send[p][t][q] for p in range(P)]) for t in range(3)] for q in range(P)]
    torch.cuda.synchronize()
    for t, x in enumerate(xs):
        want = oracle.seq_to_head(workloads.seq_shards(x, P))
        for q in range(P):
            got = bits_of(recv[q][t]).reshape(N, fs[t], d)
            assert np.array_equal(got, want[q][:, los[t]:los[t] + fs[t]]), (t, q)
    # the way back: rank q's fragment rows of rank p go to p, which unpacks them
    out = [[torch.zeros_like(seq[t][p]) for t in range(3)] for p in range(P)]
    for p in range(P):
        back = [torch.stack([recv[q][t].reshape(N, fs[t], d)[p * n:(p + 1) * n] for q in range(P)])
                for t in range(3)]
        U.ulysses_a2a_unpack(*back, *out[p], N, P, H, H_kv, d, lo, f)
    torch.cuda.synchronize()
    for t, x in enumerate(xs):
        hx = x.shape[1]
        hl = hx // P
        cols = np.zeros(hx, dtype=bool)
        for q in range(P):
            cols[q * hl + los[t]: q * hl + los[t] + fs[t]] = True
        for p in range(P):
            got = bits_of(out[p][t])
            src = workloads.seq_shards(x, P)[p]
            assert np.array_equal(got[:, cols], src[:, cols]), (t, p)
            assert not got[:, ~cols].any(), (t, p)           # untouched columns stay zero


def test_pack_validation():
    import ulysses_sequence_parallelism_b200 as U
    x = torch.empty(64, 8, 64, dtype=torch.bfloat16, device="cuda")
    s = torch.empty(2, 64, 2, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(U.UlyssesError):      # chunk of 3 heads: not whole GQA groups of 2
        U.ulysses_a2a_pack(x, None, None, s, None, None, 128, 2, 8, 4, 64, 0, 3)
    with pytest.raises(U.UlyssesError):      # chunk past the rank's 4 heads
        U.ulysses_a2a_pack(x, None, None, s, None, None, 128, 2, 8, 4, 64, 2, 4)


def _free_port():
    with socket.socket() as s_:
        s_.bind(("127.0.0.1", 0))
        return s_.getsockname()[1]


def test_dist_layer_single_process_nccl_matches_oracle_and_layer():
    import torch.distributed as dist
    import ulysses_sequence_parallelism_b200 as U
    N, H, H_kv, d = 640, 8, 2, 128
    cu_np = np.array([0, 1, 200, 513, 640], dtype=np.int32)
    q, k, v, do = (_draw(s, 40 + i) for i, s in enumerate([(N, H, d), (N, H_kv, d), (N, H_kv, d), (N, H, d)]))
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        cu = torch.tensor(cu_np, device="cuda")
        layer = U.UlyssesDistLayer(N, H, H_kv, d, cu_seqlens=cu, chunk_heads=4, deterministic=True)
        assert len(layer.plan.chunks) == 2
        o = layer.forward(to_dev(q), to_dev(k), to_dev(v))
        dq, dk, dv = layer.backward(to_dev(do))
        torch.cuda.synchronize()
        assert U.ulysses_get_device_status() == (0, 0)
        ref = U.UlyssesLayer(N, 1, H, H_kv, d, cu_seqlens=cu, deterministic=True)
        o1 = ref.forward([to_dev(q)], [to_dev(k)], [to_dev(v)])
        g1 = ref.backward([to_dev(do)])
        torch.cuda.synchronize()
        for a, b in zip((o, dq, dk, dv), (o1[0], *[x[0] for x in g1])):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16))
        w = oracle.widen_bf16
        o_r, _ = oracle.attention_forward(w(q), w(k), w(v), cu_np)
        g_r = oracle.attention_backward(w(q), w(k), w(v), w(do), cu_np)
        assert_close("O", f64(o), o_r)
        for name, a, b in zip(("dQ", "dK", "dV"), (dq, dk, dv), g_r):
            assert_close(name, f64(a), b)
    finally:
        dist.destroy_process_group()
