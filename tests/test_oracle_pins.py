"""Pins for the CPU oracle, against things other than the oracle itself:
hand-derived closed forms (tests/golden/), a pure-Python brute force, central
finite differences, exact invariants of the method (permute then inverse is
the identity; the result does not depend on P; Ulysses equals plain attention
on the unsharded tensors) and special cases of softmax attention.
All CPU, all small."""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import attention as oatt
from oracle.brute import brute_attention, brute_seq_to_head_element
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed):
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(shape)


def _frac(a):
    return np.array([[float(Fraction(x)) for x in row] for row in a])


# --------------------------------------------------------------------------- golden
def test_golden_geometric_weights():
    g = json.load(open(os.path.join(GOLDEN, "geometric_weights.json")))
    q = np.array(g["q"], dtype=np.float64)
    k = np.zeros((4, 1, 2))
    k[:, 0, 0] = np.array(g["k_ln2_multiple"]) * math.log(2.0)
    v = np.array(g["v"], dtype=np.float64)
    for key, cu in (("causal", None), ("varlen", g["varlen"]["cu_seqlens"])):
        o, lse = oracle.attention_forward(q, k, v, cu, scale=g["scale"])
        exp = g[key]
        np.testing.assert_allclose(o[:, 0, :], _frac(exp["o"]), rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse[0], np.log([float(Fraction(x)) for x in exp["lse_exp"]]),
                                   rtol=0, atol=1e-14)


def test_golden_uniform_attention_grad():
    g = json.load(open(os.path.join(GOLDEN, "uniform_attention_grad.json")))
    k = np.array(g["k"], dtype=np.float64)
    v = np.array(g["v"], dtype=np.float64)
    do = np.array(g["do"], dtype=np.float64)
    q = np.zeros_like(k)
    o, _ = oracle.attention_forward(q, k, v, scale=g["scale"])
    dq, dk, dv = oracle.attention_backward(q, k, v, do, scale=g["scale"])
    e = g["expect"]
    np.testing.assert_allclose(o[:, 0], _frac(e["o"]), atol=1e-14, rtol=0)
    np.testing.assert_allclose(dv[:, 0], _frac(e["dv"]), atol=1e-14, rtol=0)
    np.testing.assert_allclose(dq[:, 0], _frac(e["dq"]), atol=1e-14, rtol=0)
    np.testing.assert_allclose(dk[:, 0], _frac(e["dk"]), atol=1e-14, rtol=0)


# --------------------------------------------------------------------------- brute force
@pytest.mark.parametrize("cu", [None, [0, 5, 12], [0, 1, 2, 7, 12]])
@pytest.mark.parametrize("H,H_kv", [(4, 2), (2, 2), (3, 1)])
def test_forward_matches_brute_force(cu, H, H_kv):
    N, d = 12, 8
    q, k, v = _rand((N, H, d), 1), _rand((N, H_kv, d), 2), _rand((N, H_kv, d), 3)
    o, lse = oracle.attention_forward(q, k, v, cu)
    ob, lseb = brute_attention(q.tolist(), k.tolist(), v.tolist(), cu)
    np.testing.assert_allclose(o, np.array(ob), atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, np.array(lseb), atol=1e-12, rtol=0)


def test_lse_is_log_sum_exp_of_scaled_scores():
    N, H, d = 9, 2, 4
    q, k, v = _rand((N, H, d), 4), _rand((N, 1, d), 5), _rand((N, 1, d), 6)
    _, lse = oracle.attention_forward(q, k, v, scale=0.7)
    for h in range(H):
        for i in range(N):
            s = [0.7 * math.fsum(q[i, h, c] * k[j, 0, c] for c in range(d)) for j in range(i + 1)]
            assert abs(lse[h, i] - math.log(math.fsum(math.exp(x) for x in s))) < 1e-12


# --------------------------------------------------------------------------- gradients
def _loss(q, k, v, do, cu, scale):
    o, _ = oracle.attention_forward(q, k, v, cu, scale)
    return float(np.sum(o * do))


@pytest.mark.parametrize("cu", [None, [0, 3, 10]])
def test_backward_matches_finite_differences(cu):
    N, H, H_kv, d = 10, 2, 1, 4
    q, k, v, do = _rand((N, H, d), 7), _rand((N, H_kv, d), 8), _rand((N, H_kv, d), 9), _rand((N, H, d), 10)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, cu)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = x.copy(); xp[idx] += h
            xm = x.copy(); xm[idx] -= h
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            lp = _loss(args["q"], args["k"], args["v"], do, cu, None)
            args[name] = xm
            lm = _loss(args["q"], args["k"], args["v"], do, cu, None)
            num[idx] = (lp - lm) / (2 * h)
        err = np.max(np.abs(num - g)) / max(1e-12, np.max(np.abs(g)))
        assert err < 1e-6, (name, err)


def test_dv_is_p_transpose_do_brute_force():
    N, d = 7, 3
    q, k, v, do = _rand((N, 1, d), 11), _rand((N, 1, d), 12), _rand((N, 1, d), 13), _rand((N, 1, d), 14)
    _, _, dv = oracle.attention_backward(q, k, v, do)
    sc = 1 / math.sqrt(d)
    for j in range(N):
        for c in range(d):
            acc = []
            for i in range(j, N):
                w = [math.exp(sc * sum(q[i, 0, t] * k[jj, 0, t] for t in range(d))) for jj in range(i + 1)]
                acc.append(w[j] / math.fsum(w) * do[i, 0, c])
            assert abs(dv[j, 0, c] - math.fsum(acc)) < 1e-12


def test_gradient_sums_vanish():
    """Rows of dS sum to zero, so sum_j dK_j = 0 within each document; the
    softmax weights of a row sum to one, so sum_j dV_j = sum_i dO_i."""
    N, H, H_kv, d = 24, 4, 2, 8
    cu = [0, 9, 24]
    q, k, v, do = _rand((N, H, d), 15), _rand((N, H_kv, d), 16), _rand((N, H_kv, d), 17), _rand((N, H, d), 18)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, cu)
    for a, b in zip(cu[:-1], cu[1:]):
        np.testing.assert_allclose(dk[a:b].sum(axis=0), 0.0, atol=1e-12)
        for g in range(H_kv):
            np.testing.assert_allclose(dv[a:b, g].sum(axis=0), do[a:b, 2 * g:2 * g + 2].sum(axis=(0, 1)), atol=1e-12)


def test_bwd_preprocess_is_rowwise_dot():
    o, do = _rand((5, 3, 4), 19), _rand((5, 3, 4), 20)
    D = oracle.bwd_preprocess(o, do)
    for n in range(5):
        for h in range(3):
            assert abs(D[h, n] - math.fsum(o[n, h, c] * do[n, h, c] for c in range(4))) < 1e-13


# --------------------------------------------------------------------------- special cases
def test_rows_sum_to_one_and_respect_mask():
    """With V = identity (d = N) the output row i is the softmax row p_i itself."""
    N = 10
    cu = [0, 4, 10]
    q, k = _rand((N, 1, N), 21), _rand((N, 1, N), 22)
    v = np.eye(N)[:, None, :]
    o, _ = oracle.attention_forward(q, k, v, cu)
    p = o[:, 0, :]
    np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-14)
    starts = [0] * 4 + [4] * 6
    for i in range(N):
        for j in range(N):
            if j > i or j < starts[i]:
                assert p[i, j] == 0.0
            else:
                assert p[i, j] > 0.0


def test_constant_v_gives_constant_output():
    N, H, d = 16, 2, 8
    q, k = _rand((N, H, d), 23), _rand((N, 1, d), 24)
    v = np.tile(np.arange(d, dtype=np.float64), (N, 1, 1))
    o, _ = oracle.attention_forward(q, k, v, [0, 7, 16])
    np.testing.assert_allclose(o, np.broadcast_to(np.arange(d, dtype=np.float64), o.shape), atol=1e-13)


def test_first_token_of_each_document_returns_its_value():
    N, H, d = 20, 2, 4
    cu = [0, 6, 13, 20]
    q, k, v = _rand((N, H, d), 25), _rand((N, 1, d), 26), _rand((N, 1, d), 27)
    o, lse = oracle.attention_forward(q, k, v, cu)
    sc = 1 / math.sqrt(d)
    for s in cu[:-1]:
        for h in range(H):
            assert np.array_equal(o[s, h], v[s, 0])
            assert abs(lse[h, s] - sc * float(q[s, h] @ k[s, 0])) < 1e-14


def test_large_logit_selects_argmax():
    N, d = 8, 4
    q = np.zeros((N, 1, d)); k = np.zeros((N, 1, d)); v = _rand((N, 1, d), 28)
    q[:, 0, 0] = 1.0
    k[3, 0, 0] = 200.0          # key 3 dominates every row that may see it
    o, _ = oracle.attention_forward(q, k, v)
    for i in range(3, N):
        np.testing.assert_allclose(o[i, 0], v[3, 0], atol=1e-12)


def test_gqa_reduces_to_mha_with_replicated_kv():
    N, H, d = 12, 4, 8
    q, k, v = _rand((N, H, d), 29), _rand((N, 2, d), 30), _rand((N, 2, d), 31)
    o_gqa, l_gqa = oracle.attention_forward(q, k, v, [0, 5, 12])
    krep, vrep = np.repeat(k, 2, axis=1), np.repeat(v, 2, axis=1)    # head h -> kv head h // 2
    o_mha, l_mha = oracle.attention_forward(q, krep, vrep, [0, 5, 12])
    assert np.array_equal(o_gqa, o_mha) and np.array_equal(l_gqa, l_mha)
    dq1, dk1, dv1 = oracle.attention_backward(q, k, v, o_gqa, [0, 5, 12])
    dq2, dk2, dv2 = oracle.attention_backward(q, krep, vrep, o_gqa, [0, 5, 12])
    np.testing.assert_allclose(dq1, dq2, atol=1e-13)
    np.testing.assert_allclose(dk1, dk2[:, 0::2] + dk2[:, 1::2], atol=1e-13)
    np.testing.assert_allclose(dv1, dv2[:, 0::2] + dv2[:, 1::2], atol=1e-13)


def test_varlen_single_document_equals_causal():
    N, H, d = 16, 2, 8
    q, k, v = _rand((N, H, d), 32), _rand((N, 1, d), 33), _rand((N, 1, d), 34)
    a = oracle.attention_forward(q, k, v, None)
    b = oracle.attention_forward(q, k, v, [0, N])
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_varlen_equals_per_document_concatenation():
    N, H, d = 21, 2, 8
    cu = [0, 4, 15, 21]
    q, k, v, do = _rand((N, H, d), 35), _rand((N, 1, d), 36), _rand((N, 1, d), 37), _rand((N, H, d), 38)
    o, lse = oracle.attention_forward(q, k, v, cu)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, cu)
    for a, b in zip(cu[:-1], cu[1:]):
        o2, l2 = oracle.attention_forward(q[a:b], k[a:b], v[a:b])
        np.testing.assert_allclose(o[a:b], o2, atol=1e-14)
        np.testing.assert_allclose(lse[:, a:b], l2, atol=1e-14)
        g2 = oracle.attention_backward(q[a:b], k[a:b], v[a:b], do[a:b])
        for x, y in zip((dq, dk, dv), g2):
            np.testing.assert_allclose(x[a:b], y, atol=1e-13)


# --------------------------------------------------------------------------- sampled oracles
def test_sampled_rows_and_columns_match_full():
    N, H, H_kv, d = 40, 4, 2, 8
    cu = [0, 13, 31, 40]
    q, k, v, do = _rand((N, H, d), 39), _rand((N, H_kv, d), 40), _rand((N, H_kv, d), 41), _rand((N, H, d), 42)
    o, lse = oracle.attention_forward(q, k, v, cu)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, cu)
    D = oracle.bwd_preprocess(o, do)
    rows = [0, 12, 13, 14, 30, 39, 5]
    for h in range(H):
        o_r, l_r, dq_r, D_r = oracle.attention_rows(q, k, v, h, rows, do=do, cu_seqlens=cu)
        np.testing.assert_allclose(o_r, o[rows, h], atol=1e-13)
        np.testing.assert_allclose(l_r, lse[h, rows], atol=1e-13)
        np.testing.assert_allclose(dq_r, dq[rows, h], atol=1e-13)
        np.testing.assert_allclose(D_r, D[h, rows], atol=1e-13)
    cols = [0, 12, 13, 29, 39]
    for g in range(H_kv):
        dk_c, dv_c = oracle.attention_kv_cols(q, k, v, do, g, cols, cu_seqlens=cu)
        np.testing.assert_allclose(dk_c, dk[cols, g], atol=1e-13)
        np.testing.assert_allclose(dv_c, dv[cols, g], atol=1e-13)


# --------------------------------------------------------------------------- permutes
def test_permute_matches_elementwise_definition():
    P, n, Hx, d = 4, 3, 8, 2
    x = _rand((P * n, Hx, d), 43)
    xs = workloads.seq_shards(x, P)
    xh = oracle.seq_to_head(xs)
    nested = [s.tolist() for s in xs]
    for q_rank in range(P):
        for t in range(P * n):
            for j in range(Hx // P):
                for c in range(d):
                    assert xh[q_rank][t, j, c] == brute_seq_to_head_element(nested, q_rank, t, j, c)


@pytest.mark.parametrize("P", [1, 2, 4, 8])
def test_permute_then_inverse_is_identity(P):
    x = np.arange(16 * 8 * 4, dtype=np.float64).reshape(16, 8, 4)
    xs = workloads.seq_shards(x, P)
    back = oracle.head_to_seq(oracle.seq_to_head(xs))
    for a, b in zip(xs, back):
        assert np.array_equal(a, b)


def test_permute_with_one_rank_is_identity_copy():
    x = _rand((6, 4, 2), 44)
    assert np.array_equal(oracle.seq_to_head([x])[0], x)


def test_permute_rank_range_selects_destinations():
    x = _rand((8, 8, 2), 45)
    xs = workloads.seq_shards(x, 4)
    full = oracle.seq_to_head(xs)
    part = oracle.seq_to_head(xs, 1, 3)
    assert np.array_equal(part[0], full[1]) and np.array_equal(part[1], full[2])


def test_head_shard_holds_all_positions_for_a_slice_of_heads():
    """After the first all-to-all a rank holds every token of its own head subset."""
    N, H, d, P = 8, 4, 2, 2
    x = _rand((N, H, d), 46)
    xh = oracle.seq_to_head(workloads.seq_shards(x, P))
    for q_rank in range(P):
        assert np.array_equal(xh[q_rank], x[:, q_rank * 2:(q_rank + 1) * 2])


# --------------------------------------------------------------------------- the layer
def test_layer_is_invariant_to_P_and_equals_unsharded_attention():
    N, H, H_kv, d = 32, 8, 4, 8
    cu = [0, 11, 32]
    q, k, v, do = _rand((N, H, d), 47), _rand((N, H_kv, d), 48), _rand((N, H_kv, d), 49), _rand((N, H, d), 50)
    o_ref, _ = oracle.attention_forward(q, k, v, cu)
    g_ref = oracle.attention_backward(q, k, v, do, cu)
    for P in (1, 2, 4):
        sh = lambda x: workloads.seq_shards(x, P)
        o_seq, lse_h = oracle.ulysses_layer_forward(sh(q), sh(k), sh(v), cu)
        o = np.concatenate(o_seq, axis=0)
        np.testing.assert_allclose(o, o_ref, atol=1e-14)
        grads = oracle.ulysses_layer_backward(sh(q), sh(k), sh(v), sh(do), cu)
        for g, r in zip(grads, g_ref):
            np.testing.assert_allclose(np.concatenate(g, axis=0), r, atol=1e-13)
        if P == 1:
            o_p1, g_p1 = o, [np.concatenate(g, axis=0) for g in grads]
        else:   # identical per-head arithmetic on every P: bit-identical results
            assert np.array_equal(o, o_p1)
            for g, r in zip(grads, g_p1):
                assert np.array_equal(np.concatenate(g, axis=0), r)


# --------------------------------------------------------------------------- mutations
def test_pins_catch_planted_mistakes(monkeypatch):
    """Plant plausible mistakes in the oracle (on the CPU) and check that the
    brute-force pin rejects each one."""
    N, H, H_kv, d = 9, 4, 2, 4
    cu = [0, 4, 9]
    q, k, v = _rand((N, H, d), 51), _rand((N, H_kv, d), 52), _rand((N, H_kv, d), 53)
    ob, lb = brute_attention(q.tolist(), k.tolist(), v.tolist(), cu)
    ob, lb = np.array(ob), np.array(lb)

    def differs():
        o, l = oracle.attention_forward(q, k, v, cu)
        return not (np.allclose(o, ob, atol=1e-9) and np.allclose(l, lb, atol=1e-9))

    assert not differs()
    orig_starts = oatt.doc_starts
    monkeypatch.setattr(oatt, "doc_starts", lambda n, c=None: orig_starts(n, None))   # drop varlen
    assert differs()
    monkeypatch.setattr(oatt, "doc_starts", orig_starts)
    monkeypatch.setattr(oatt, "_scale", lambda d_, s: 1.0)                               # wrong scale
    assert differs()


# ---------------------------------------------------------------- projections (NEXT-4)

def _brute_matvec(x_row, w):
    """Pure-Python y_j = fsum_c x_c w[j][c]."""
    import math
    return [math.fsum(float(a) * float(b) for a, b in zip(x_row, w_row)) for w_row in w]


def test_qkv_projection_matches_brute_force_and_splits_heads_in_order():
    import oracle
    rng = np.random.Generator(np.random.PCG64(71))
    P, n, hidden, H, H_kv, d = 2, 3, 5, 4, 2, 2
    x_seq = [rng.standard_normal((n, hidden)) for _ in range(P)]
    w = rng.standard_normal(((H + 2 * H_kv) * d, hidden))
    q, k, v = oracle.qkv_projection(x_seq, w, H, H_kv, d)
    for p in range(P):
        for s in range(n):
            y = _brute_matvec(x_seq[p][s], w)
            for h in range(H):
                assert np.allclose(q[p][s, h], y[h * d:(h + 1) * d], rtol=0, atol=1e-12)
            for h in range(H_kv):
                assert np.allclose(k[p][s, h], y[(H + h) * d:(H + h + 1) * d], rtol=0, atol=1e-12)
                assert np.allclose(v[p][s, h], y[(H + H_kv + h) * d:(H + H_kv + h + 1) * d], rtol=0, atol=1e-12)


def test_qkv_projection_selection_weights_route_inputs():
    """W_qkv made of unit rows picks input features: Q head h dim c must be
    x[(h*d + c) % hidden], K and V shifted by 1 and 2: pins row order and the
    head/dim reshape (a transposed or mis-split W fails)."""
    import oracle
    P, n, H, H_kv, d = 2, 4, 4, 2, 3
    hidden = 7
    rng = np.random.Generator(np.random.PCG64(72))
    x_seq = [rng.standard_normal((n, hidden)) for _ in range(P)]
    rows = (H + 2 * H_kv) * d
    w = np.zeros((rows, hidden))
    src = []
    for r in range(rows):
        shift = 0 if r < H * d else (1 if r < (H + H_kv) * d else 2)
        c = (r + shift) % hidden
        w[r, c] = 1.0
        src.append(c)
    q, k, v = oracle.qkv_projection(x_seq, w, H, H_kv, d)
    for p in range(P):
        for h in range(H):
            for c in range(d):
                assert np.array_equal(q[p][:, h, c], x_seq[p][:, src[h * d + c]])
        for h in range(H_kv):
            for c in range(d):
                assert np.array_equal(k[p][:, h, c], x_seq[p][:, src[(H + h) * d + c]])
                assert np.array_equal(v[p][:, h, c], x_seq[p][:, src[(H + H_kv + h) * d + c]])


def test_out_projection_identity_and_brute_force():
    import oracle
    rng = np.random.Generator(np.random.PCG64(73))
    P, n, H, d = 2, 3, 2, 3
    o_seq = [rng.standard_normal((n, H, d)) for _ in range(P)]
    y = oracle.out_projection(o_seq, np.eye(H * d))
    for p in range(P):
        assert np.array_equal(y[p], o_seq[p].reshape(n, H * d))        # identity: heads concatenated in order
    w = rng.standard_normal((5, H * d))
    y = oracle.out_projection(o_seq, w)
    for p in range(P):
        for s in range(n):
            assert np.allclose(y[p][s], _brute_matvec(o_seq[p][s].reshape(-1), w), rtol=0, atol=1e-12)


def test_projection_planted_transpose_is_caught():
    """A plausible mistake (x @ w instead of x @ w.T, on a square W) must fail
    the brute-force pin above."""
    rng = np.random.Generator(np.random.PCG64(74))
    x = rng.standard_normal((3, 4))
    w = rng.standard_normal((4, 4))
    wrong = x @ w
    right = np.array([_brute_matvec(r, w) for r in x])
    assert not np.allclose(wrong, right, atol=1e-6)


def test_projection_gradients_match_directional_derivatives():
    """The projections are linear, so for L = sum_t <y_t, g_t> the change of L
    along any direction E of an input or weight equals <gradient, E> exactly
    (up to fp64 rounding): pins both backward formulas, including which side
    of W each product takes and the head order of g."""
    import oracle
    rng = np.random.Generator(np.random.PCG64(75))
    P, n, hidden, H, H_kv, d = 2, 3, 6, 4, 2, 2
    x = [rng.standard_normal((n, hidden)) for _ in range(P)]
    w = rng.standard_normal(((H + 2 * H_kv) * d, hidden))
    gq = [rng.standard_normal((n, H, d)) for _ in range(P)]
    gk = [rng.standard_normal((n, H_kv, d)) for _ in range(P)]
    gv = [rng.standard_normal((n, H_kv, d)) for _ in range(P)]

    def L(xs, ws):
        q, k, v = oracle.qkv_projection(xs, ws, H, H_kv, d)
        return sum(np.sum(a * b) for t, g in ((q, gq), (k, gk), (v, gv)) for a, b in zip(t, g))

    dx, dw = oracle.qkv_projection_backward(x, w, gq, gk, gv)
    Ew = rng.standard_normal(w.shape)
    Ex = [rng.standard_normal(a.shape) for a in x]
    eps = 1.0                       # exact for a linear map
    assert abs((L(x, w + eps * Ew) - L(x, w)) - np.sum(dw * Ew)) < 1e-9
    assert abs((L([a + eps * e for a, e in zip(x, Ex)], w) - L(x, w)) -
               sum(np.sum(a * e) for a, e in zip(dx, Ex))) < 1e-9

    o = [rng.standard_normal((n, H, d)) for _ in range(P)]
    wo = rng.standard_normal((hidden, H * d))
    gy = [rng.standard_normal((n, hidden)) for _ in range(P)]

    def Lo(os_, ws):
        return sum(np.sum(a * b) for a, b in zip(oracle.out_projection(os_, ws), gy))

    do, dwo = oracle.out_projection_backward(o, wo, gy)
    Ewo = rng.standard_normal(wo.shape)
    Eo = [rng.standard_normal(a.shape) for a in o]
    assert abs((Lo(o, wo + Ewo) - Lo(o, wo)) - np.sum(dwo * Ewo)) < 1e-9
    assert abs((Lo([a + e for a, e in zip(o, Eo)], wo) - Lo(o, wo)) - sum(np.sum(a * e) for a, e in zip(do, Eo))) < 1e-9


def test_projection_gradients_brute_force():
    import math
    import oracle
    rng = np.random.Generator(np.random.PCG64(76))
    n, hidden, H, d = 2, 3, 2, 2
    o = [rng.standard_normal((n, H, d))]
    wo = rng.standard_normal((hidden, H * d))
    gy = [rng.standard_normal((n, hidden))]
    do, dwo = oracle.out_projection_backward(o, wo, gy)
    for t in range(n):
        for f in range(H * d):
            want = math.fsum(gy[0][t, k] * wo[k, f] for k in range(hidden))
            assert abs(do[0].reshape(n, -1)[t, f] - want) < 1e-12
    for k in range(hidden):
        for f in range(H * d):
            want = math.fsum(gy[0][t, k] * o[0].reshape(n, -1)[t, f] for t in range(n))
            assert abs(dwo[k, f] - want) < 1e-12


def test_widen_bf16_is_exact_on_every_bit_pattern():
    """bf16 -> fp64 widening against torch's own bf16 -> float64 conversion on
    all 65,536 bit patterns (finite values equal exactly; +-inf and NaN land in
    the same classes), a few values fixed by the format (1, -2, the largest
    finite value, the smallest subnormal), and the round trip through the
    input generator's float32 -> bf16 rounding."""
    import torch
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ours = oracle.widen_bf16(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    fin = np.isfinite(ref)
    assert fin.sum() == 65536 - 2 * 128                   # exponent field all ones: 2 signs x 128 mantissas
    assert np.array_equal(ours[fin], ref[fin])
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    assert np.array_equal(np.isposinf(ours), np.isposinf(ref)) and np.array_equal(np.isneginf(ours), np.isneginf(ref))
    w = lambda b: float(oracle.widen_bf16(np.array([b], dtype=np.uint16))[0])
    assert w(0x3F80) == 1.0 and w(0xC000) == -2.0 and w(0x0000) == 0.0
    assert w(0x7F7F) == (2.0 - 2.0 ** -7) * 2.0 ** 127
    assert w(0x0001) == 2.0 ** -133
    assert w(0x3F81) == 1.0 + 2.0 ** -7                   # one bf16 step above 1 (7 stored mantissa bits)
    back = workloads.round_to_bf16_bits(ours[fin].astype(np.float32))
    assert np.array_equal(back, bits[fin])
