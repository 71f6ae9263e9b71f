"""The Ulysses all-to-alls as index arithmetic (test infrastructure only).

Method: before attention an all-to-all gives each rank the whole sequence for
a subset of the heads; after attention a second all-to-all undoes it
(theaicatchup.com, "How Does Ulysses Sequence Parallelism Actually Work?";
two all-to-alls per layer also in contenidos2-1ml.pages.dev, "¿Qué es Ulysses
y por qué importa?").

Layouts (the pages fix none; plainest reading):
  sequence shard of rank p : [N/P, Hx, d], global token t = p*N/P + s
  head shard of rank q     : [N, Hx/P, d], local head j = global head q*Hx/P + j
Every element moves once; nothing is computed, so the result is exact.
"""
from typing import List, Optional

import numpy as np


def seq_to_head(x_seq: List[np.ndarray], rank_lo: int = 0, rank_hi: Optional[int] = None) -> List[np.ndarray]:
    """All-to-all #1. ``x_seq[p]`` is rank p's ``[N/P, Hx, d]`` shard; returns,
    for each destination rank q in [rank_lo, rank_hi), ``[N, Hx/P, d]`` with
    ``out[q][t, j] = x_seq[t // (N/P)][t % (N/P), q*Hx/P + j]``."""
    P = len(x_seq)
    n, Hx, d = x_seq[0].shape
    assert Hx % P == 0
    Hl = Hx // P
    rank_hi = P if rank_hi is None else rank_hi
    out = []
    for q in range(rank_lo, rank_hi):
        dst = np.empty((n * P, Hl, d), dtype=x_seq[0].dtype)
        for p in range(P):           # source rank p contributes tokens [p*n, (p+1)*n)
            dst[p * n:(p + 1) * n] = x_seq[p][:, q * Hl:(q + 1) * Hl]
        out.append(dst)
    return out


def head_to_seq(x_head: List[np.ndarray]) -> List[np.ndarray]:
    """All-to-all #2, the inverse of ``seq_to_head``. ``x_head[q]`` is rank q's
    ``[N, Hx/P, d]``; returns rank p's ``[N/P, Hx, d]`` with
    ``out[p][s, q*Hx/P + j] = x_head[q][p*N/P + s, j]``."""
    P = len(x_head)
    N, Hl, d = x_head[0].shape
    assert N % P == 0
    n = N // P
    out = []
    for p in range(P):
        dst = np.empty((n, Hl * P, d), dtype=x_head[0].dtype)
        for q in range(P):
            dst[:, q * Hl:(q + 1) * Hl] = x_head[q][p * n:(p + 1) * n]
        out.append(dst)
    return out
