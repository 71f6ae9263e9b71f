"""Head fragmentation (q2bstudio.com, "Ulysses Unleashed: Context Parallelism
with Fragmentation by Heads"): a rank processes its heads a few GQA groups at a
time. The fragment permutes are bit copies checked against the oracle's
all-to-all restricted to the fragment's heads; the fragmented layer must give
exactly the unfragmented layer's results (heads never interact)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_util import shards_to_dev, f64, assert_close

pytestmark = pytest.mark.gpu


def _bits(shape, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.integers(0, 1 << 16, size=shape, dtype=np.uint16) & np.uint16(0x7F7F)


def _dev(a):
    return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)


@pytest.mark.parametrize("N,P,H,H_kv,d,h_lo,f", [
    (512, 2, 8, 2, 128, 4, 4),      # rank 1's whole head set (one GQA group of 4)
    (384, 4, 16, 4, 64, 8, 4),      # rank 2, one group
    (256, 2, 16, 8, 128, 2, 4),     # two groups of 2 inside rank 0
    (1024, 1, 8, 8, 128, 3, 1),     # P = 1, MHA, a single head
])
def test_fragment_permutes_bit_exact(N, P, H, H_kv, d, h_lo, f):
    import ulysses_sequence_parallelism_b200 as U
    g = H // H_kv
    n = N // P
    xs = [_bits((N, H, d), 1), _bits((N, H_kv, d), 2), _bits((N, H_kv, d), 3)]
    seqs = [[_dev(x[p * n:(p + 1) * n]) for p in range(P)] for x in xs]
    fq = torch.empty(N, f, d, dtype=torch.bfloat16, device="cuda")
    fk = torch.empty(N, f // g, d, dtype=torch.bfloat16, device="cuda")
    fv = torch.empty_like(fk)
    U.ulysses_a2a_seq_to_head_frag(seqs[0], seqs[1], seqs[2], fq, fk, fv, N, P, H, H_kv, d, h_lo, f)
    torch.cuda.synchronize()
    for x, got, lo, cnt in ((xs[0], fq, h_lo, f), (xs[1], fk, h_lo // g, f // g), (xs[2], fv, h_lo // g, f // g)):
        full = np.concatenate(oracle.seq_to_head(workloads.seq_shards(x, P)), axis=1)   # [N, Hx, d]
        ref = full[:, lo:lo + cnt]
        assert np.array_equal(got.view(torch.int16).cpu().numpy().view(np.uint16), ref)
    # inverse: writes exactly the fragment's columns of the sequence shards
    outs = [[_dev(np.full_like(x[p * n:(p + 1) * n], 0x1234)) for p in range(P)] for x in xs]
    U.ulysses_a2a_head_to_seq_frag(fq, fk, fv, outs[0], outs[1], outs[2], N, P, H, H_kv, d, h_lo, f)
    torch.cuda.synchronize()
    for x, o, lo, cnt in ((xs[0], outs[0], h_lo, f), (xs[1], outs[1], h_lo // g, f // g),
                          (xs[2], outs[2], h_lo // g, f // g)):
        got = np.concatenate([t.view(torch.int16).cpu().numpy().view(np.uint16) for t in o], axis=0)
        want = np.full_like(x, 0x1234)
        want[:, lo:lo + cnt] = x[:, lo:lo + cnt]
        assert np.array_equal(got, want)


def _layer_run(q, k, v, do, P, cu, **kw):
    import ulysses_sequence_parallelism_b200 as U
    N, H, d = q.shape
    H_kv = k.shape[1]
    cu_t = None if cu is None else torch.tensor(np.asarray(cu, np.int32), device="cuda")
    layer = U.UlyssesLayer(N, P, H, H_kv, d, cu_seqlens=cu_t, **kw)
    o = layer.forward(shards_to_dev(q, P), shards_to_dev(k, P), shards_to_dev(v, P))
    g = layer.backward(shards_to_dev(do, P))
    torch.cuda.synchronize()
    assert U.ulysses_get_device_status() == (0, 0)
    cat = lambda ts: torch.cat(ts, 0).view(torch.int16).cpu().numpy()
    return {"o": cat(o), "lse": np.concatenate([l.cpu().numpy() for l in layer.lse], 0),
            "dq": cat(g[0]), "dk": cat(g[1]), "dv": cat(g[2])}


@pytest.mark.parametrize("deterministic", [True, False], ids=["twopass", "onepass"])
@pytest.mark.parametrize("frag", [2, 4])
def test_fragmented_layer_equals_unfragmented(frag, deterministic):
    N, P, H, H_kv, d = 1024, 2, 8, 4, 128
    cu = [0, 200, 201, 700, 1024]
    rng = np.random.Generator(np.random.PCG64(31))
    mk = lambda s: workloads.round_to_bf16_bits(rng.standard_normal(s, dtype=np.float32))
    q, k, v, do = mk((N, H, d)), mk((N, H_kv, d)), mk((N, H_kv, d)), mk((N, H, d))
    a = _layer_run(q, k, v, do, P, cu, deterministic=deterministic)
    b = _layer_run(q, k, v, do, P, cu, deterministic=deterministic, head_fragment=frag)
    for n in ("o", "lse", "dk", "dv") + (("dq",) if deterministic else ()):
        assert np.array_equal(a[n], b[n]), n
    if not deterministic:
        w = lambda x: x.view(np.uint16).astype(np.uint32) << 16
        fa, fb = (w(x[("dq")]).view(np.float32).astype(np.float64) for x in (a, b))
        assert np.all(np.abs(fa - fb) <= np.abs(fa) * 2.0 ** -7 + 1e-5 * np.abs(fa).max())


def test_fragmented_layer_matches_oracle():
    N, P, H, H_kv, d = 512, 2, 8, 2, 64
    cu = [0, 100, 512]
    rng = np.random.Generator(np.random.PCG64(37))
    mk = lambda s: workloads.round_to_bf16_bits(rng.standard_normal(s, dtype=np.float32))
    q, k, v, do = mk((N, H, d)), mk((N, H_kv, d)), mk((N, H_kv, d)), mk((N, H, d))
    got = _layer_run(q, k, v, do, P, cu, head_fragment=4)
    w = oracle.widen_bf16
    sh = lambda x: workloads.seq_shards(w(x), P)
    o_ref, _ = oracle.ulysses_layer_forward(sh(q), sh(k), sh(v), cu)
    g_ref = oracle.ulysses_layer_backward(sh(q), sh(k), sh(v), sh(do), cu)
    wid = lambda bits: w(bits.view(np.uint16))
    assert_close("O", wid(got["o"]), np.concatenate(o_ref, 0))
    for name, ref in zip(("dq", "dk", "dv"), g_ref):
        assert_close(name, wid(got[name]), np.concatenate(ref, 0))
