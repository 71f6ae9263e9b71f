"""The N > 1 paths on CPU with world_size-2 gloo process groups.

1. bench.py's whole-job throughput: every rank runs its own layer, the
   slowest rank's time sets the job time, value = all ranks' tokens / that time.
2. The method's real exchange: on P processes the first all-to-all is a
   collective (each rank sends head block q of its token chunk to rank q). Done
   here with torch.distributed.all_to_all_single over gloo on CPU, it must give
   exactly the oracle's single-process index-arithmetic permute (the layout the
   one-GPU emulation produces), and the inverse exchange must restore the
   sequence shards.
"""
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


def _init(rank, world, port):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))


def _worker_aggregate(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    _init(rank, world, port)
    from bench import aggregate_over_ranks

    def reduce_max(x):
        t = torch.tensor([x], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    local_ms = [10.0, 12.5][rank]
    ms, val = aggregate_over_ranks(local_ms, 65536, world, reduce_max)
    q.put((rank, ms, val))
    dist.destroy_process_group()


def _worker_all_to_all(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    _init(rank, world, port)
    import oracle
    import workloads
    N, H, d = 64, 8, 4
    x = np.arange(N * H * d, dtype=np.float64).reshape(N, H, d)
    n, Hl = N // world, H // world
    mine = torch.from_numpy(np.ascontiguousarray(workloads.seq_shards(x, world)[rank]))   # [n, H, d]
    # send head block q of my tokens to rank q: pack as [world, n, Hl, d]
    send = mine.view(n, world, Hl, d).permute(1, 0, 2, 3).contiguous()
    recv = torch.empty_like(send)                     # [world(source p), n, Hl, d]
    dist.all_to_all_single(recv, send)
    head = recv.reshape(N, Hl, d)                      # tokens of source p come in order p
    ref = oracle.seq_to_head(workloads.seq_shards(x, world))[rank]
    ok1 = np.array_equal(head.numpy(), ref)
    # inverse exchange
    back_send = head.view(world, n, Hl, d).contiguous()
    back_recv = torch.empty_like(back_send)            # [world(source q), n, Hl, d]
    dist.all_to_all_single(back_recv, back_send)
    seq = back_recv.permute(1, 0, 2, 3).reshape(n, H, d)
    ok2 = np.array_equal(seq.numpy(), mine.numpy())
    q.put((rank, ok1, ok2))
    dist.destroy_process_group()


def _run(fn, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=fn, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(out)


def test_bench_throughput_is_max_over_ranks():
    out = _run(_worker_aggregate)
    for rank, ms, val in out:
        assert ms == 12.5                              # the slower rank sets the job time
        assert abs(val - 2 * 65536 / 0.0125) < 1e-6    # both ranks' tokens


def test_real_all_to_all_equals_emulated_permute():
    out = _run(_worker_all_to_all)
    for rank, ok1, ok2 in out:
        assert ok1, f"rank {rank}: all_to_all result differs from the seq->head permute"
        assert ok2, f"rank {rank}: inverse exchange did not restore the shard"
