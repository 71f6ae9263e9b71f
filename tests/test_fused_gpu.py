"""The fused layer (the all-to-alls folded into the attention kernels'
addressing: ulysses_attn_fwd_seq / ulysses_attn_bwd_seq) against the three-call
path it replaces: bit-identical O, LSE, dQ, dK, dV with the two-pass backward,
since the kernels do the same arithmetic in the same order and only fetch and
store elsewhere; with the one-pass backward everything but dQ (whose fp32 sums
run in timing-dependent order). One case is also checked against the fp64
oracle directly."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_util import shards_to_dev, f64, assert_close, err_stats, LSE_MAX_ABS

pytestmark = pytest.mark.gpu


def _draw(N, H, H_kv, d, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    mk = lambda s: workloads.round_to_bf16_bits(rng.standard_normal(s, dtype=np.float32))
    return mk((N, H, d)), mk((N, H_kv, d)), mk((N, H_kv, d)), mk((N, H, d))


def _run(q, k, v, do, P, cu, fused, deterministic=False):
    import ulysses_sequence_parallelism_b200 as U
    N, H, d = q.shape
    H_kv = k.shape[1]
    cu_t = None if cu is None else torch.tensor(np.asarray(cu, np.int32), device="cuda")
    layer = U.UlyssesLayer(N, P, H, H_kv, d, cu_seqlens=cu_t, fused=fused, deterministic=deterministic)
    o = layer.forward(shards_to_dev(q, P), shards_to_dev(k, P), shards_to_dev(v, P))
    g = layer.backward(shards_to_dev(do, P))
    torch.cuda.synchronize()
    assert U.ulysses_get_device_status() == (0, 0)
    cat = lambda ts: torch.cat(ts, 0).view(torch.int16).cpu().numpy()
    return {"o": cat(o), "lse": np.concatenate([l.cpu().numpy() for l in layer.lse], 0),
            "dq": cat(g[0]), "dk": cat(g[1]), "dv": cat(g[2])}


CASES = [
    (512, 2, 8, 8, 64, None),
    (1024, 4, 16, 4, 128, [0, 300, 301, 777, 1024]),
    (1024, 8, 16, 8, 128, None),            # 128 tokens per shard, one kv head per rank
    (2048, 1, 4, 1, 128, [0, 100, 1500, 2048]),
    (1536, 4, 8, 4, 64, [0, 1, 640, 1536]),
]


@pytest.mark.parametrize("deterministic", [True, False], ids=["twopass", "onepass"])
@pytest.mark.parametrize("N,P,H,H_kv,d,cu", CASES)
def test_fused_layer_is_bit_identical_to_three_calls(N, P, H, H_kv, d, cu, deterministic):
    q, k, v, do = _draw(N, H, H_kv, d, seed=N + P + d)
    a = _run(q, k, v, do, P, cu, fused=False, deterministic=deterministic)
    b = _run(q, k, v, do, P, cu, fused=True, deterministic=deterministic)
    for n in ("o", "lse", "dq", "dk", "dv"):
        if n == "dq" and not deterministic and d == 128:
            wa = a[n].view(np.uint16).astype(np.uint32) << 16
            wb = b[n].view(np.uint16).astype(np.uint32) << 16
            fa, fb = wa.view(np.float32).astype(np.float64), wb.view(np.float32).astype(np.float64)
            assert np.all(np.abs(fa - fb) <= np.abs(fa) * 2.0 ** -7 + 1e-5 * np.abs(fa).max()), n
        else:
            assert np.array_equal(a[n], b[n]), n


def test_fused_layer_matches_oracle():
    N, P, H, H_kv, d = 1024, 4, 8, 4, 128
    cu = [0, 250, 900, 1024]
    q, k, v, do = _draw(N, H, H_kv, d, seed=5)
    b = _run(q, k, v, do, P, cu, fused=True)
    w = oracle.widen_bf16
    sh = lambda x: workloads.seq_shards(w(x), P)
    o_ref, lse_ref = oracle.ulysses_layer_forward(sh(q), sh(k), sh(v), cu)
    g_ref = oracle.ulysses_layer_backward(sh(q), sh(k), sh(v), sh(do), cu)
    wid = lambda bits: w(bits.view(np.uint16))
    assert_close("O", wid(b["o"]), np.concatenate(o_ref, 0))
    assert err_stats(b["lse"].astype(np.float64), np.concatenate(lse_ref, 0))[0] <= LSE_MAX_ABS
    for name, x, r in zip(("dQ", "dK", "dV"), ("dq", "dk", "dv"), g_ref):
        assert_close(name, wid(b[x]), np.concatenate(r, 0))


def test_fused_forward_rank_range_writes_only_its_heads():
    import ulysses_sequence_parallelism_b200 as U
    N, P, H, H_kv, d = 1024, 4, 8, 4, 64
    q, k, v, _ = _draw(N, H, H_kv, d, seed=9)
    qs, ks, vs = shards_to_dev(q, P), shards_to_dev(k, P), shards_to_dev(v, P)
    full = [torch.empty(N // P, H, d, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    lse = [torch.empty(H // P, N, dtype=torch.float32, device="cuda") for _ in range(P)]
    U.ulysses_attn_fwd_seq(qs, ks, vs, full, lse, N, P, H, H_kv, d)
    part = [torch.full((N // P, H, d), 7.0, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    lse2 = [torch.empty(H // P, N, dtype=torch.float32, device="cuda") for _ in range(P)]
    U.ulysses_attn_fwd_seq(qs, ks, vs, part, lse2, N, P, H, H_kv, d, rank_lo=1, rank_hi=3)
    torch.cuda.synchronize()
    Hl = H // P
    for p in range(P):
        assert torch.equal(part[p][:, Hl:3 * Hl], full[p][:, Hl:3 * Hl])
        assert torch.all(part[p][:, :Hl] == 7.0) and torch.all(part[p][:, 3 * Hl:] == 7.0)
    for r in (1, 2):
        assert torch.equal(lse2[r], lse[r])


@pytest.mark.parametrize("rank_lo,rank_hi", [(0, 4), (1, 3)])
def test_seq_backward_staged_and_direct_agree(rank_lo, rank_hi):
    """ulysses_attn_bwd_seq with the larger workspace stages Q and dO in head
    shards first; with the plain workspace it streams them from the sequence
    shards. Both must give the same dK, dV bits (dQ to one bf16 step: fp32
    sums in timing order), for all ranks and for a rank range (whose heads
    alone are written)."""
    import ulysses_sequence_parallelism_b200 as U
    N, P, H, H_kv, d = 1024, 4, 8, 4, 128
    cu = torch.tensor([0, 300, 301, 777, 1024], dtype=torch.int32, device="cuda")
    q, k, v, do = _draw(N, H, H_kv, d, seed=31)
    qs, ks, vs, dos = (shards_to_dev(x, P) for x in (q, k, v, do))
    o = [torch.empty(N // P, H, d, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    lse = [torch.empty(H // P, N, dtype=torch.float32, device="cuda") for _ in range(P)]
    U.ulysses_attn_fwd_seq(qs, ks, vs, o, lse, N, P, H, H_kv, d, cu)
    res = []
    for size in (U.ulysses_attn_bwd_seq_workspace_size, U.ulysses_attn_bwd_workspace_size):
        ws = torch.empty(size(N, P, H, H_kv, d, False), dtype=torch.uint8, device="cuda")
        g = [[torch.full((N // P, hx, d), 3.0, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
             for hx in (H, H_kv, H_kv)]
        U.ulysses_attn_bwd_seq(qs, ks, vs, o, lse, dos, *g, N, P, H, H_kv, d, ws, cu,
                               rank_lo=rank_lo, rank_hi=rank_hi)
        torch.cuda.synchronize()
        assert U.ulysses_get_device_status() == (0, 0)
        res.append(g)
    staged, direct = res
    for t, name in enumerate(("dq", "dk", "dv")):
        hl = (H if t == 0 else H_kv) // P
        cols = slice(rank_lo * hl, rank_hi * hl)
        for p in range(P):
            a, b = staged[t][p], direct[t][p]
            assert torch.all(a[:, :rank_lo * hl] == 3.0) and torch.all(a[:, rank_hi * hl:] == 3.0), name
            if name == "dq":
                fa, fb = a[:, cols].float(), b[:, cols].float()
                assert torch.all((fa - fb).abs() <= fb.abs() * 2.0 ** -7 + 1e-5 * fb.abs().max()), name
            else:
                assert torch.equal(a[:, cols], b[:, cols]), name
