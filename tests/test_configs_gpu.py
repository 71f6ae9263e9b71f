"""GPU parity on the five workloads at their full sizes, in the launch
configuration bench.py times (the UlyssesLayer path).

The oracle computes, exactly in fp64, sampled outputs it can afford one by
one: O, LSE and dQ of sampled query rows (each depends only on its own row),
and dK/dV of key positions near the end of each document (each needs only the
rows after it). The tiny workload is checked in full. Properties that hold at
any size are checked on the whole output: sum_j dV_j = sum_i dO_i per
document and kv head, and sum_j dK_j ~ 0 per document and kv head."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.gpu_util import (to_dev, f64, shards_to_dev, assert_close, LSE_MAX_ABS, err_stats, sample_rows,
                            tail_cols)

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


def _check_sampled(w, inp, res, n_rows):
    N, P, H, H_kv, d = w.N, w.P, w.H, w.H_kv, w.d
    group = H // H_kv
    cu = inp["cu_seqlens"]
    rows = sample_rows(N, P, cu, n_rows)
    cols = tail_cols(N, cu, per_doc=16) if w.backward else []
    widen = oracle.widen_bf16
    for g in range(H_kv):
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
            if not w.rank_sequential:
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


@pytest.mark.parametrize("name,n_rows", [("llama8k", 96), ("varlen64k", 64), ("long96k", 48)])
def test_workload_sampled(name, n_rows):
    w = workloads.get(name)
    inp = workloads.generate(w)
    res = _run(w, inp)
    _check_sampled(w, inp, res, n_rows)
    _check_sums(w, inp, res)


def test_million_token_rank_sequential_sampled():
    w = workloads.get("million")
    inp = workloads.generate(w)
    res = _run(w, inp)
    _check_sampled(w, inp, res, 12)
