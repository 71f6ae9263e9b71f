"""The projections on either side of the Ulysses exchange (test infrastructure only).

Every rank projects Q, K and V for its own chunk of tokens before the first
all-to-all, and projects the attention output on its own shard after the
second (theaicatchup.com, "How Does Ulysses Sequence Parallelism Actually
Work?"; contenidos2-1ml.pages.dev, "¿Qué es Ulysses y por qué importa?").
Plain fp64 matrix products per token:
  [q_t | k_t | v_t] = x_t W_qkv^T,  W_qkv rows: H query heads of d, then H_kv
  key heads, then H_kv value heads (head-major, d contiguous);
  y_t = o_t W_o^T,  o_t = the token's H heads of d concatenated in head order.
"""
from typing import List

import numpy as np


def qkv_projection(x_seq: List[np.ndarray], w_qkv: np.ndarray, H: int, H_kv: int, d: int):
    """Sequence shards x_seq[p] [N/P, hidden] -> sequence-sharded (Q, K, V):
    lists of [N/P, H, d], [N/P, H_kv, d], [N/P, H_kv, d]."""
    q_seq, k_seq, v_seq = [], [], []
    for x in x_seq:
        y = np.asarray(x, np.float64) @ np.asarray(w_qkv, np.float64).T
        n = y.shape[0]
        q_seq.append(y[:, :H * d].reshape(n, H, d))
        k_seq.append(y[:, H * d:(H + H_kv) * d].reshape(n, H_kv, d))
        v_seq.append(y[:, (H + H_kv) * d:].reshape(n, H_kv, d))
    return q_seq, k_seq, v_seq


def out_projection(o_seq: List[np.ndarray], w_o: np.ndarray) -> List[np.ndarray]:
    """Sequence-sharded O [N/P, H, d] -> Y [N/P, hidden] per shard."""
    out = []
    for o in o_seq:
        n = o.shape[0]
        out.append(np.asarray(o, np.float64).reshape(n, -1) @ np.asarray(w_o, np.float64).T)
    return out
