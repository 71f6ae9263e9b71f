"""fp64 causal softmax attention, forward and backward (test infrastructure only).

What it computes (per head: the method runs ordinary attention on each head by
itself, since the heads do not interact -- theaicatchup.com, citing the
DeepSpeed-Ulysses paper in "How Does Ulysses Sequence Parallelism Actually
Work?"; the Spanish note stresses that Ulysses leaves the attention arithmetic
itself unchanged -- contenidos2-1ml.pages.dev, "Conclusión rápida"):

  s_ij  = scale * (q_i . k_j)            for allowed j, scale = 1/sqrt(d)
  allowed(i, j)  <=>  j <= i  and  doc(j) == doc(i)
  p_ij  = exp(s_ij) / sum_allowed exp(s_ij')
  o_i   = sum_j p_ij v_j,   lse_i = ln sum_allowed exp(s_ij)

Query head h reads key/value head h // (H/H_kv) (grouped-query attention with
consecutive groups).  Documents come from ``cu_seqlens`` (packed variable
length sequences, which the pages say need their own flag and no padding --
theaicatchup.com, "Best practices" and "Can You Integrate Ulysses...").

Backward (the pages train with it but do not write it; standard calculus of
the forward above), with loss gradient dO:
  dV_j = sum_i p_ij dO_i
  dP_ij = dO_i . v_j
  dS_ij = p_ij (dP_ij - sum_j' p_ij' dP_ij')
  dQ_i = scale sum_j dS_ij k_j,   dK_j = scale sum_i dS_ij q_i
with dK/dV of a key/value head summed over the query heads that read it.

Rows are processed in blocks only to bound memory: each row's softmax is
taken over its whole allowed set in one step (no online rescaling); masked
columns outside [doc start, i] are simply not formed.
"""
from typing import Optional, Sequence

import numpy as np


def _scale(d: int, scale: Optional[float]) -> float:
    return 1.0 / np.sqrt(d) if (scale is None or scale <= 0) else float(scale)


def doc_starts(N: int, cu_seqlens=None) -> np.ndarray:
    """First token of the document that contains each token."""
    if cu_seqlens is None:
        return np.zeros(N, dtype=np.int64)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    idx = np.searchsorted(cu, np.arange(N), side="right") - 1
    return cu[idx]


def doc_ends(N: int, cu_seqlens=None) -> np.ndarray:
    """One past the last token of the document that contains each token."""
    if cu_seqlens is None:
        return np.full(N, N, dtype=np.int64)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    idx = np.searchsorted(cu, np.arange(N), side="right") - 1
    return cu[idx + 1]


def _softmax_rows(q_rows, k_cols, rows, cols, start, scale):
    """Full-row softmax of the allowed scores: returns (p, lse)."""
    s = (q_rows @ k_cols.T) * scale
    allowed = (cols[None, :] <= rows[:, None]) & (cols[None, :] >= start[rows][:, None])
    s = np.where(allowed, s, -np.inf)
    m = s.max(axis=1)
    e = np.exp(s - m[:, None])
    l = e.sum(axis=1)
    return e / l[:, None], m + np.log(l)


def attention_forward(q, k, v, cu_seqlens=None, scale=None, row_block: int = 512):
    """q [N,H,d], k/v [N,H_kv,d] fp64 -> (o [N,H,d], lse [H,N])."""
    N, H, d = q.shape
    H_kv = k.shape[1]
    assert H % H_kv == 0
    group = H // H_kv
    sc = _scale(d, scale)
    start = doc_starts(N, cu_seqlens)
    o = np.zeros((N, H, d))
    lse = np.zeros((H, N))
    for h in range(H):
        g = h // group
        for r0 in range(0, N, row_block):
            rows = np.arange(r0, min(N, r0 + row_block))
            c0, c1 = int(start[rows].min()), int(rows[-1]) + 1
            cols = np.arange(c0, c1)
            p, l = _softmax_rows(q[rows, h], k[c0:c1, g], rows, cols, start, sc)
            o[rows, h] = p @ v[c0:c1, g]
            lse[h, rows] = l
    return o, lse


def bwd_preprocess(o, do):
    """D_i = sum_c dO_ic * O_ic per (token, head): [N,H,d] x2 -> [H,N]."""
    return np.einsum("nhc,nhc->hn", do, o)


def attention_backward(q, k, v, do, cu_seqlens=None, scale=None, row_block: int = 512):
    """Gradients of sum(O * dO) w.r.t. q, k, v (fp64)."""
    N, H, d = q.shape
    H_kv = k.shape[1]
    group = H // H_kv
    sc = _scale(d, scale)
    start = doc_starts(N, cu_seqlens)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for h in range(H):
        g = h // group
        for r0 in range(0, N, row_block):
            rows = np.arange(r0, min(N, r0 + row_block))
            c0, c1 = int(start[rows].min()), int(rows[-1]) + 1
            cols = np.arange(c0, c1)
            p, _ = _softmax_rows(q[rows, h], k[c0:c1, g], rows, cols, start, sc)
            dv[c0:c1, g] += p.T @ do[rows, h]
            dp = do[rows, h] @ v[c0:c1, g].T
            ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))
            dq[rows, h] = sc * (ds @ k[c0:c1, g])
            dk[c0:c1, g] += sc * (ds.T @ q[rows, h])
    return dq, dk, dv


def attention_rows(q, k, v, h: int, rows: Sequence[int], do=None, cu_seqlens=None,
                   scale=None, row_block: int = 64):
    """Exact per-row outputs for query head ``h`` at the given rows only:
    (o [R,d], lse [R], dq [R,d] or None, D [R] or None). Each row depends on
    its own allowed keys only, so no other row is needed; D_i uses the
    oracle's own o_i."""
    N, H, d = q.shape
    group = H // k.shape[1]
    g = h // group
    sc = _scale(d, scale)
    start = doc_starts(N, cu_seqlens)
    rows = np.asarray(rows, dtype=np.int64)
    R = len(rows)
    o = np.zeros((R, d))
    lse = np.zeros(R)
    dq = None if do is None else np.zeros((R, d))
    D = None if do is None else np.zeros(R)
    order = np.argsort(rows)
    for b0 in range(0, R, row_block):
        sel = order[b0:b0 + row_block]
        rr = rows[sel]
        c0, c1 = int(start[rr].min()), int(rr.max()) + 1
        cols = np.arange(c0, c1)
        kk = k[c0:c1, g]
        vv = v[c0:c1, g]
        p, l = _softmax_rows(q[rr, h], kk, rr, cols, start, sc)
        o[sel] = p @ vv
        lse[sel] = l
        if do is not None:
            dp = do[rr, h] @ vv.T
            ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))
            dq[sel] = sc * (ds @ kk)
            D[sel] = np.einsum("rc,rc->r", do[rr, h], o[sel])
    return o, lse, dq, D


def attention_kv_cols(q, k, v, do, g: int, cols: Sequence[int], cu_seqlens=None,
                      scale=None, row_block: int = 256):
    """Exact dK, dV of key/value head ``g`` at the given key positions only
    (summed over the query heads of its group). Key j receives gradient from
    every row i >= j of its document, so all those rows are formed in full;
    cheap when the sampled keys sit near the end of their documents."""
    N, H, d = q.shape
    group = H // k.shape[1]
    sc = _scale(d, scale)
    start = doc_starts(N, cu_seqlens)
    end = doc_ends(N, cu_seqlens)
    cols = np.asarray(cols, dtype=np.int64)
    need = np.zeros(N, dtype=bool)
    for j in cols:
        need[j:end[j]] = True
    need_rows = np.nonzero(need)[0]
    dk = np.zeros((len(cols), d))
    dv = np.zeros((len(cols), d))
    for h in range(g * group, (g + 1) * group):
        for b0 in range(0, len(need_rows), row_block):
            rr = need_rows[b0:b0 + row_block]
            c0, c1 = int(start[rr].min()), int(rr.max()) + 1
            ccols = np.arange(c0, c1)
            kk = k[c0:c1, g]
            vv = v[c0:c1, g]
            p, _ = _softmax_rows(q[rr, h], kk, rr, ccols, start, sc)
            dp = do[rr, h] @ vv.T
            ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))
            inb = (cols >= c0) & (cols < c1)
            if not inb.any():
                continue
            jj = cols[inb] - c0
            dv[inb] += p[:, jj].T @ do[rr, h]
            dk[inb] += sc * (ds[:, jj].T @ q[rr, h])
    return dk, dv
