"""GPU parity on the five workloads at their full sizes, in the launch
configuration bench.py times (the UlyssesLayer path).

The oracle computes, exactly in fp64, what it can afford:
  - every output of whole GQA groups (a kv head and its query heads: heads do
    not interact, so a group is an exact sub-problem): O, LSE, dQ, dK, dV of
    kv head 0 (rank 0) and of the last kv head (rank P-1) at the 8K and the
    packed 64K workloads, element by element;
  - O, LSE and dQ of sampled query rows on every head (each row depends only
    on its own keys);
  - dK/dV of key positions near the end of each document, and at the 96K
    workload of every tile edge (+-1) and seeded keys across its last 4096
    positions (each key needs only the rows after it, which the oracle forms
    in full).
The tiny workload is checked in full. The million-token workload checks its
rank-sequential permutes bit for bit, every rank's LSE and O on sampled rows.
Properties that hold at any size are checked on the whole output:
sum_j dV_j = sum_i dO_i per document and kv head, and sum_j dK_j ~ 0."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_util import (to_dev, f64, bits_of, shards_to_dev, assert_close, LSE_MAX_ABS, err_stats,
                            sample_rows, tail_cols)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _cu_dev(cu):
    return None if cu is None else torch.tensor(cu, dtype=torch.int32, device="cuda")


def _run(w, inp):
    import ulysses_sequence_parallelism_b200 as U
    P, H, H_kv, d, N = w.P, w.H, w.H_kv, w.d, w.N
    cu = inp["cu_seqlens"]
    layer = U.UlyssesLayer(N, P, H, H_kv, d, cu_seqlens=_cu_dev(cu), backward=w.backward,
                           rank_sequential=w.rank_sequential)
    o = layer.forward(shards_to_dev(inp["q"], P), shards_to_dev(inp["k"], P), shards_to_dev(inp["v"], P))
    res = {"layer": layer, "o_seq": o}
    if w.backward:
        res["grads"] = layer.backward(shards_to_dev(inp["do"], P))
    torch.cuda.synchronize()
    code, word = U.ulysses_get_device_status()
    assert code == 0 and word == 0
    return res


def _rows_of(seq_list, rows, h):
    """Gather global rows of head h from sequence shards (on device) -> fp64."""
    n = seq_list[0].shape[0]
    idx = torch.tensor(rows, device="cuda")
    allr = torch.cat([x[:, h] for x in seq_list], dim=0) if len(seq_list) > 1 else seq_list[0][:, h]
    return f64(allr.index_select(0, idx))


def _check_sampled(w, inp, res, n_rows, extra_cols=()):
    N, P, H, H_kv, d = w.N, w.P, w.H, w.H_kv, w.d
    group = H // H_kv
    cu = inp["cu_seqlens"]
    rows = sample_rows(N, P, cu, n_rows)
    tail = tail_cols(N, cu, per_doc=16) if w.backward else []
    widen = oracle.widen_bf16
    for g in range(H_kv):
        # the costlier extra key columns only for kv head 0 (rank 0) and the last one (rank P-1)
        cols = sorted(set(tail) | set(extra_cols)) if (w.backward and g in (0, H_kv - 1)) else tail
        k_g = widen(inp["k"][:, g:g + 1])
        v_g = widen(inp["v"][:, g:g + 1])
        q_grp = np.zeros((N, group, d))   # only the rows the oracle needs are filled
        do_grp = np.zeros((N, group, d)) if w.backward else None
        need = sorted(set(rows) | set(c2 for c in cols for c2 in range(c, oracle.doc_ends(N, cu)[c])))
        need = np.asarray(need, dtype=np.int64)
        q_grp[need] = widen(inp["q"][need, g * group:(g + 1) * group])
        if w.backward:
            do_grp[need] = widen(inp["do"][need, g * group:(g + 1) * group])
        for hh in range(group):
            h = g * group + hh
            o_r, lse_r, dq_r, _ = oracle.attention_rows(
                q_grp[:, hh:hh + 1], k_g, v_g, 0, rows,
                do=None if do_grp is None else do_grp[:, hh:hh + 1], cu_seqlens=cu)
            assert_close(f"O head {h}", _rows_of(res["o_seq"], rows, h), o_r)
            r, hl = divmod(h, H // P)
            lse_gpu = res["layer"].lse[r][hl].index_select(0, torch.tensor(rows, device="cuda"))
            ma, _ = err_stats(lse_gpu.cpu().numpy().astype(np.float64), lse_r)
            assert ma <= LSE_MAX_ABS, f"LSE head {h}: {ma:.3e}"
            if w.backward:
                assert_close(f"dQ head {h}", _rows_of(res["grads"][0], rows, h), dq_r)
        if w.backward:
            # dK/dV of kv head g summed over its query heads: the group is H = group, H_kv = 1
            dk_c, dv_c = oracle.attention_kv_cols(q_grp, k_g, v_g, do_grp, 0, cols, cu_seqlens=cu)
            assert_close(f"dK kv head {g}", _rows_of(res["grads"][1], cols, g), dk_c)
            assert_close(f"dV kv head {g}", _rows_of(res["grads"][2], cols, g), dv_c)


def _check_sums(w, inp, res):
    """sum over a document's keys of dV = sum over its rows of dO (per kv head,
    over the group); sum of dK over a document ~ 0."""
    N, P, H, H_kv, d = w.N, w.P, w.H, w.H_kv, w.d
    group = H // H_kv
    cu = inp["cu_seqlens"] if inp["cu_seqlens"] is not None else np.array([0, N])
    dq, dk, dv = (torch.cat(x, dim=0).double() for x in res["grads"])
    do = torch.cat(shards_to_dev(inp["do"], P), dim=0).double()
    for a, b in zip(cu[:-1], cu[1:]):
        a, b = int(a), int(b)
        sdv = dv[a:b].sum(0)                                 # [H_kv, d]
        sdo = do[a:b].view(b - a, H_kv, group, d).sum((0, 2))
        scale_ref = dv[a:b].abs().sum(0).max().item() + 1e-30
        assert (sdv - sdo).abs().max().item() <= 2e-2 * scale_ref + 5e-2
        sdk = dk[a:b].sum(0)
        assert (sdk.abs().max().item()) <= 2e-2 * (dk[a:b].abs().sum(0).max().item() + 1e-30) + 5e-2


def test_tiny_full():
    w = workloads.get("tiny")
    inp = workloads.generate(w)
    res = _run(w, inp)
    qs, ks, vs = (workloads.seq_shards(oracle.widen_bf16(inp[t]), w.P) for t in ("q", "k", "v"))
    o_ref, lse_ref = oracle.ulysses_layer_forward(qs, ks, vs, None)
    assert_close("O", np.concatenate([f64(x) for x in res["o_seq"]], 0), np.concatenate(o_ref, 0))
    for r in range(w.P):
        ma, _ = err_stats(res["layer"].lse[r].cpu().numpy().astype(np.float64), lse_ref[r])
        assert ma <= LSE_MAX_ABS


def _check_group_full(w, inp, res, g):
    """Every output of kv head g's GQA group against the fp64 oracle run on
    that group alone: O, LSE and dQ of its H/H_kv query heads on every row, and
    dK, dV of kv head g on every key."""
    N, P, H, H_kv, d = w.N, w.P, w.H, w.H_kv, w.d
    group = H // H_kv
    cu = inp["cu_seqlens"]
    widen = oracle.widen_bf16
    heads = slice(g * group, (g + 1) * group)
    q, k, v = widen(inp["q"][:, heads]), widen(inp["k"][:, g:g + 1]), widen(inp["v"][:, g:g + 1])
    do = widen(inp["do"][:, heads])
    o_ref, lse_ref = oracle.attention_forward(q, k, v, cu)
    dq_ref, dk_ref, dv_ref = oracle.attention_backward(q, k, v, do, cu)
    cat = lambda xs, sl: f64(torch.cat([x[:, sl] for x in xs], dim=0))
    assert_close(f"O kv group {g}", cat(res["o_seq"], heads), o_ref)
    assert_close(f"dQ kv group {g}", cat(res["grads"][0], heads), dq_ref)
    assert_close(f"dK kv head {g}", cat(res["grads"][1], slice(g, g + 1)), dk_ref)
    assert_close(f"dV kv head {g}", cat(res["grads"][2], slice(g, g + 1)), dv_ref)
    hl_per = H // P
    for hh in range(group):
        h = g * group + hh
        r, hl = divmod(h, hl_per)
        ma, _ = err_stats(res["layer"].lse[r][hl].cpu().numpy().astype(np.float64), lse_ref[hh])
        assert ma <= LSE_MAX_ABS, f"LSE head {h}: {ma:.3e}"


@pytest.mark.parametrize("name", ["llama8k", "varlen64k"])
def test_workload_full_gqa_groups(name):
    """Element-wise parity of whole GQA groups at full size: kv head 0 (held by
    rank 0) and the last kv head (held by rank P-1)."""
    w = workloads.get(name)
    inp = workloads.generate(w)
    res = _run(w, inp)
    for g in (0, w.H_kv - 1):
        _check_group_full(w, inp, res, g)


@pytest.mark.parametrize("name,n_rows", [("llama8k", 96), ("varlen64k", 64), ("long96k", 48)])
def test_workload_sampled(name, n_rows):
    w = workloads.get(name)
    inp = workloads.generate(w)
    res = _run(w, inp)
    extra = ()
    if name == "long96k":
        # one 96K-token sequence: keys across its last 4096 positions (every tile
        # edge +-1 and seeded ones) each gather gradient from up to 4096 rows x 4 heads
        rng = np.random.Generator(np.random.PCG64(96))
        lo = w.N - 4096
        edges = [e + o for e in range(lo, w.N, 128) for o in (-1, 0, 1) if lo <= e + o < w.N]
        extra = sorted(set(edges) | set(int(x) for x in rng.integers(lo, w.N, size=32)))
    _check_sampled(w, inp, res, n_rows, extra_cols=extra)
    _check_sums(w, inp, res)


def test_million_token_rank_sequential():
    """The million-token workload (P = 8, ranks one after another): each rank's
    seq->head permute of Q, K and V equals the oracle's all-to-all bit for bit
    over the whole head shard, and the head->seq permute of those shards
    rebuilds the sequence shards exactly; then the layer's forward matches the
    oracle on sampled rows of every head, LSE included for every rank."""
    import ulysses_sequence_parallelism_b200 as U
    w = workloads.get("million")
    inp = workloads.generate(w)
    N, P, H, H_kv, d = w.N, w.P, w.H, w.H_kv, w.d
    res = _run(w, inp)
    layer = res["layer"]
    seq = {t: shards_to_dev(inp[t], P) for t in ("q", "k", "v")}
    back = {t: [torch.zeros_like(x) for x in seq[t]] for t in seq}
    host_shards = {t: workloads.seq_shards(inp[t], P) for t in seq}
    for r in range(P):
        rb = lambda b: [b[0] if i == r else None for i in range(P)]
        U.ulysses_a2a_seq_to_head(seq["q"], seq["k"], seq["v"], rb(layer.q_h), rb(layer.k_h), rb(layer.v_h), N, P,
                                  H, H_kv, d, rank_lo=r, rank_hi=r + 1)
        for t, buf in (("q", layer.q_h[0]), ("k", layer.k_h[0]), ("v", layer.v_h[0])):
            want = oracle.seq_to_head(host_shards[t], rank_lo=r, rank_hi=r + 1)[0]
            assert np.array_equal(bits_of(buf), want), f"rank {r} {t}: seq->head permute differs"
        U.ulysses_a2a_head_to_seq(rb(layer.q_h), rb(layer.k_h), rb(layer.v_h),
                                  back["q"], back["k"], back["v"], N, P, H, H_kv, d, rank_lo=r, rank_hi=r + 1)
    torch.cuda.synchronize()
    for t in seq:
        for p in range(P):
            assert torch.equal(back[t][p].view(torch.int16), seq[t][p].view(torch.int16)), f"{t} shard {p}"
    del back, seq
    _check_sampled(w, inp, res, 64)
