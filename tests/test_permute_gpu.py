"""GPU parity for the two all-to-all permutes: bit-exact against the oracle's
index arithmetic, inverse-then-forward identity, rank ranges, and guard
canaries around every rank buffer (out-of-bounds writes would change them)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_util import to_dev, bits_of

pytestmark = pytest.mark.gpu

CANARY = 2048          # bf16 elements (4 KB) of sentinel on each side of every rank buffer
SENTINEL = -12345


def padded(shape):
    """A rank buffer living inside a bigger tensor with sentinel pads on both sides."""
    n = int(np.prod(shape))
    big = torch.full((n + 2 * CANARY,), SENTINEL, dtype=torch.int16, device="cuda")
    view = big[CANARY:CANARY + n].view(torch.bfloat16).view(*shape)
    return big, view


def pads_intact(big):
    h = big.cpu().numpy()
    return bool(np.all(h[:CANARY] == SENTINEL) and np.all(h[-CANARY:] == SENTINEL))


def rand_bits(shape, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.integers(0, 1 << 16, size=shape, dtype=np.uint16) & np.uint16(0x7F7F)   # finite patterns


def run_seq_to_head(U, seqs, P, H, H_kv, d, lo=0, hi=None):
    N = seqs[0][0].shape[0] * P
    hi = P if hi is None else hi
    outs, bigs = [], []
    for t, x in enumerate(seqs):
        hx = x[0].shape[1]
        bufs = []
        for r in range(P):
            if lo <= r < hi:
                b, v = padded((N, hx // P, d))
                bigs.append(b)
                bufs.append(v)
            else:
                bufs.append(None)
        outs.append(bufs)
    x0, x1, x2 = (seqs + [None, None])[:3]
    o0, o1, o2 = (outs + [None, None])[:3]
    U.ulysses_a2a_seq_to_head(x0, x1, x2, o0, o1, o2, N, P, H, H_kv, d, rank_lo=lo, rank_hi=hi)
    torch.cuda.synchronize()
    assert all(pads_intact(b) for b in bigs), "canary overwritten"
    return outs


SHAPES = [
    (512, 2, 8, 8, 64),        # tiny workload shape
    (1024, 4, 32, 8, 128),     # Llama heads
    (96, 1, 4, 2, 64),         # P = 1: identity copy
    (64, 4, 4, 4, 128),        # P = H: one head per rank
    (200, 8, 16, 8, 64),       # 25 tokens per rank, 1 kv head per rank
    (48, 2, 6, 2, 64),         # 3 query heads per rank
]


@pytest.mark.parametrize("N,P,H,H_kv,d", SHAPES)
def test_seq_to_head_and_back_bit_exact(N, P, H, H_kv, d):
    import ulysses_sequence_parallelism_b200 as U
    q, k, v = rand_bits((N, H, d), 1), rand_bits((N, H_kv, d), 2), rand_bits((N, H_kv, d), 3)
    seqs = [[to_dev(s) for s in workloads.seq_shards(x, P)] for x in (q, k, v)]
    heads = run_seq_to_head(U, seqs, P, H, H_kv, d)
    for x, got in zip((q, k, v), heads):
        ref = oracle.seq_to_head(workloads.seq_shards(x, P))
        for r in range(P):
            assert np.array_equal(bits_of(got[r]), ref[r])
    # inverse: head -> seq into padded buffers, must give back the inputs bit for bit
    backs, bigs = [], []
    for x in (q, k, v):
        hx = x.shape[1]
        bufs = []
        for r in range(P):
            b, vv = padded((N // P, hx, d))
            bigs.append(b)
            bufs.append(vv)
        backs.append(bufs)
    U.ulysses_a2a_head_to_seq(heads[0], heads[1], heads[2], backs[0], backs[1], backs[2], N, P, H, H_kv, d)
    torch.cuda.synchronize()
    assert all(pads_intact(b) for b in bigs)
    for x, got in zip((q, k, v), backs):
        for r, s in enumerate(workloads.seq_shards(x, P)):
            assert np.array_equal(bits_of(got[r]), s)


def test_single_tensor_slot_and_rank_ranges():
    import ulysses_sequence_parallelism_b200 as U
    N, P, H, H_kv, d = 256, 4, 8, 4, 128
    q = rand_bits((N, H, d), 4)
    qs = [to_dev(s) for s in workloads.seq_shards(q, P)]
    ref = oracle.seq_to_head(workloads.seq_shards(q, P))
    for lo, hi in ((0, 1), (1, 3), (3, 4)):
        out = run_seq_to_head(U, [qs], P, H, H_kv, d, lo, hi)[0]
        for r in range(lo, hi):
            assert np.array_equal(bits_of(out[r]), ref[r])
    # head -> seq from one source rank writes only that rank's head columns
    heads = [to_dev(x) for x in ref]
    dst = [torch.zeros(N // P, H, d, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    U.ulysses_a2a_head_to_seq(heads, None, None, dst, None, None, N, P, H, H_kv, d, rank_lo=2, rank_hi=3)
    torch.cuda.synchronize()
    for r, s in enumerate(workloads.seq_shards(q, P)):
        got = bits_of(dst[r])
        assert np.array_equal(got[:, 4:6], s[:, 4:6])
        assert np.all(got[:, :4] == 0) and np.all(got[:, 6:] == 0)


@pytest.mark.parametrize("name", ["tiny", "llama8k", "varlen64k", "long96k"])
def test_workload_permutes_bit_exact(name):
    import ulysses_sequence_parallelism_b200 as U
    w = workloads.get(name)
    inp = workloads.generate(w, with_do=False)
    P, H, H_kv, d, N = w.P, w.H, w.H_kv, w.d, w.N
    seqs = [[to_dev(s) for s in workloads.seq_shards(inp[t], P)] for t in ("q", "k", "v")]
    heads = [[torch.empty(N, hx // P, d, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
             for hx in (H, H_kv, H_kv)]
    U.ulysses_a2a_seq_to_head(*seqs, *heads, N, P, H, H_kv, d)
    torch.cuda.synchronize()
    for t, got in zip(("q", "k", "v"), heads):
        ref = oracle.seq_to_head(workloads.seq_shards(inp[t], P))
        for r in range(P):
            assert np.array_equal(bits_of(got[r]), ref[r]), (t, r)
    back = [[torch.empty_like(x) for x in s] for s in seqs]
    U.ulysses_a2a_head_to_seq(*heads, *back, N, P, H, H_kv, d)
    torch.cuda.synchronize()
    for s, b in zip(seqs, back):
        for x, y in zip(s, b):
            assert torch.equal(x.view(torch.int16), y.view(torch.int16))
