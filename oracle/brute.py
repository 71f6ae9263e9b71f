"""Pure-Python triple-loop attention for tiny inputs (test infrastructure only).

Written independently of ``attention.py`` (no numpy linear algebra, math.fsum
sums, explicit index tests) so that it can pin the vectorised oracle: the two
share only the definition of masked softmax attention with grouped key/value
heads (see ``attention.py``'s docstring for the citations).
"""
import math


def brute_attention(q, k, v, cu_seqlens=None, scale=None):
    """q: nested lists [N][H][d]; k, v: [N][H_kv][d]. Returns (o [N][H][d], lse [H][N])."""
    N, H, d = len(q), len(q[0]), len(q[0][0])
    H_kv = len(k[0])
    sc = 1.0 / math.sqrt(d) if (scale is None or scale <= 0) else scale
    doc = [0] * N
    if cu_seqlens is not None:
        for t in range(N):
            for m in range(len(cu_seqlens) - 1):
                if cu_seqlens[m] <= t < cu_seqlens[m + 1]:
                    doc[t] = m
    o = [[[0.0] * d for _ in range(H)] for _ in range(N)]
    lse = [[0.0] * N for _ in range(H)]
    for h in range(H):
        g = (h * H_kv) // H
        for i in range(N):
            js = [j for j in range(N) if j <= i and doc[j] == doc[i]]
            s = {j: sc * math.fsum(q[i][h][c] * k[j][g][c] for c in range(d)) for j in js}
            mx = max(s.values())
            w = {j: math.exp(s[j] - mx) for j in js}
            z = math.fsum(w.values())
            lse[h][i] = mx + math.log(z)
            for c in range(d):
                o[i][h][c] = math.fsum(w[j] * v[j][g][c] for j in js) / z
    return o, lse


def brute_seq_to_head_element(x_seq, q_rank, t, j, c):
    """One element of the seq->head all-to-all, by the definition."""
    P = len(x_seq)
    n = len(x_seq[0])
    Hl = len(x_seq[0][0]) // P
    return x_seq[t // n][t % n][q_rank * Hl + j][c]
