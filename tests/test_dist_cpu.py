"""The multi-process exchange (UlyssesDistLayer) on CPU process groups.

World size 2 with gloo: each process holds one rank's sequence shards and the
layer's exchange plan runs as on GPUs (pack, asynchronous all_to_all_single,
attention on the received head fragment, all-to-all back, unpack; two head
chunks, inbound exchanges issued before the first attention). The four local
steps are host implementations written here (index copies for pack/unpack,
the fp64 oracle for attention, rounded to bf16), so what is checked is the
exchange itself: the fragments each rank receives equal, bit for bit, the
oracle's all-to-all restricted to the chunk's heads, and the layer's outputs
and gradients equal the oracle's single-process layer bit for bit (both sides
round the same fp64 values once to bf16)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class HostKernels:
    """Host stand-ins for the library's four local steps (test only)."""

    @staticmethod
    def _slots(plan):
        return [(plan.H, plan.chunks, 1), (plan.H_kv, plan.chunks, plan.g), (plan.H_kv, plan.chunks, plan.g)]

    @staticmethod
    def pack(plan, c, x0, x1, x2, s0, s1, s2):
        for (hx, chunks, div), x, s in zip(HostKernels._slots(plan), (x0, x1, x2), (s0, s1, s2)):
            if x is None:
                continue
            lo, f = chunks[c][0] // div, chunks[c][1] // div
            hl = hx // plan.P
            s.copy_(x.view(plan.n, plan.P, hl, plan.d)[:, :, lo:lo + f].permute(1, 0, 2, 3))

    @staticmethod
    def unpack(plan, c, r0, r1, r2, x0, x1, x2):
        for (hx, chunks, div), r, x in zip(HostKernels._slots(plan), (r0, r1, r2), (x0, x1, x2)):
            if r is None:
                continue
            lo, f = chunks[c][0] // div, chunks[c][1] // div
            hl = hx // plan.P
            x.view(plan.n, plan.P, hl, plan.d)[:, :, lo:lo + f].copy_(r.permute(1, 0, 2, 3))

    @staticmethod
    def attn_fwd(plan, q, k, v, o, lse, cu, scale):
        import oracle
        w = lambda t: t.double().numpy()
        o_, l_ = oracle.attention_forward(w(q), w(k), w(v), cu)
        o.copy_(torch.from_numpy(o_).to(torch.bfloat16))
        lse.copy_(torch.from_numpy(l_).float())

    @staticmethod
    def attn_bwd(plan, q, k, v, o, lse, do, dq, dk, dv, ws, cu, scale, deterministic):
        import oracle
        w = lambda t: t.double().numpy()
        g = oracle.attention_backward(w(q), w(k), w(v), w(do), cu)
        for dst, src in zip((dq, dk, dv), g):
            dst.copy_(torch.from_numpy(src).to(torch.bfloat16))

    @staticmethod
    def workspace_bytes(plan, deterministic):
        return 1


def _worker(rank, world, port, q_out, N, H, H_kv, d, cu):
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import oracle
    import workloads
    from ulysses_sequence_parallelism_b200.dist import UlyssesDistLayer
    rng = np.random.Generator(np.random.PCG64(5))
    mk = lambda s: workloads.round_to_bf16_bits(rng.standard_normal(s, dtype=np.float32))
    q, k, v, do = mk((N, H, d)), mk((N, H_kv, d)), mk((N, H_kv, d)), mk((N, H, d))
    P, n = world, N // world
    bf = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    mine = lambda bits: bf(workloads.seq_shards(bits, P)[rank]).clone()
    layer = UlyssesDistLayer(N, H, H_kv, d, device="cpu", cu_seqlens=cu, kernels=HostKernels)
    o = layer.forward(mine(q), mine(k), mine(v))
    res = {"chunks": len(layer.plan.chunks)}
    # 1. the received head fragments are the oracle's all-to-all, chunk by chunk
    ok = True
    for c, (lo, f) in enumerate(layer.plan.chunks):
        for i, (x, hx) in enumerate(((q, H), (k, H_kv), (v, H_kv))):
            div = 1 if i == 0 else H // H_kv
            want = oracle.seq_to_head(workloads.seq_shards(x, P))[rank][:, lo // div:(lo + f) // div]
            got = layer.frag[c][i].view(torch.int16).numpy().view(np.uint16)
            ok &= bool(np.array_equal(got, want))
    res["frag"] = ok
    # 2. outputs and gradients equal the single-process oracle layer
    wd = oracle.widen_bf16
    sh = lambda bits: workloads.seq_shards(wd(bits), P)
    o_ref, _ = oracle.ulysses_layer_forward(sh(q), sh(k), sh(v), cu)
    rnd = lambda a: torch.from_numpy(a).to(torch.bfloat16).view(torch.int16)
    res["o"] = bool(torch.equal(o.view(torch.int16), rnd(o_ref[rank])))
    dq, dk, dv = layer.backward(mine(do))
    g_ref = oracle.ulysses_layer_backward(sh(q), sh(k), sh(v), sh(do), cu)
    res["grads"] = all(bool(torch.equal(a.view(torch.int16), rnd(b[rank]))) for a, b in zip((dq, dk, dv), g_ref))
    q_out.put((rank, res))
    dist.destroy_process_group()


def _run(world, *args):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q) + args) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(out, key=lambda x: x[0])


@pytest.mark.parametrize("N,H,H_kv,d,cu", [
    (64, 8, 4, 8, None),                          # 2 ranks x 4 heads = 2 chunks of one GQA group each
    (96, 8, 2, 4, [0, 5, 40, 41, 96]),            # GQA 4:1, one chunk, documents straddling the ranks
])
def test_dist_layer_exchange_matches_oracle(N, H, H_kv, d, cu):
    cu = None if cu is None else np.asarray(cu, dtype=np.int32)
    for rank, res in _run(2, N, H, H_kv, d, cu):
        assert res["frag"], f"rank {rank}: received head fragments differ from the oracle's all-to-all"
        assert res["o"], f"rank {rank}: O differs from the oracle layer"
        assert res["grads"], f"rank {rank}: gradients differ from the oracle layer"


def test_exchange_plan_chunks():
    from ulysses_sequence_parallelism_b200.dist import ExchangePlan
    p = ExchangePlan(65536, 4, 32, 8, 128)
    assert p.chunks == [(0, 4), (4, 4)] and p.send_shape(False) == (4, 16384, 4, 128)
    assert p.send_shape(True) == (4, 16384, 1, 128) and p.fragment_shape(False) == (65536, 4, 128)
    assert ExchangePlan(1 << 20, 8, 32, 8, 128).chunks == [(0, 4)]       # one GQA group per rank: one chunk
    assert ExchangePlan(8192, 2, 32, 8, 128, chunk_heads=4).chunks == [(0, 4), (4, 4), (8, 4), (12, 4)]
    steps = p.forward_steps()
    # every inbound exchange is issued before the first attention, unpacks come last
    assert steps.index(("attn", 0)) > max(steps.index(("a2a_in", c)) for c in range(2))
    assert steps[-2:] == [("unpack", 0), ("unpack", 1)]
    with pytest.raises(ValueError):
        ExchangePlan(8192, 4, 32, 8, 128, chunk_heads=2)                 # not whole GQA groups
    with pytest.raises(ValueError):
        ExchangePlan(8192, 4, 32, 8, 128, chunk_heads=12)                # does not divide H/P
