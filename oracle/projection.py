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


def qkv_projection_backward(x_seq: List[np.ndarray], w_qkv: np.ndarray, dq_seq, dk_seq, dv_seq):
    """Gradient of qkv_projection: with g_t = [dq_t | dk_t | dv_t] (each head's d
    values in head order), dx_t = g_t W_qkv and dW_qkv = sum_t g_t^T x_t.
    Returns (dx_seq list [N/P, hidden], dW_qkv)."""
    w = np.asarray(w_qkv, np.float64)
    dx, dw = [], np.zeros_like(w)
    for x, dq, dk, dv in zip(x_seq, dq_seq, dk_seq, dv_seq):
        n = x.shape[0]
        g = np.concatenate([np.asarray(t, np.float64).reshape(n, -1) for t in (dq, dk, dv)], axis=1)
        dx.append(g @ w)
        dw += g.T @ np.asarray(x, np.float64)
    return dx, dw


def out_projection_backward(o_seq: List[np.ndarray], w_o: np.ndarray, dy_seq: List[np.ndarray]):
    """Gradient of out_projection: do_t = dy_t W_o (reshaped to [H, d]) and
    dW_o = sum_t dy_t^T o_t. Returns (do_seq list [N/P, H, d], dW_o)."""
    w = np.asarray(w_o, np.float64)
    do, dw = [], np.zeros_like(w)
    for o, dy in zip(o_seq, dy_seq):
        n = o.shape[0]
        dy = np.asarray(dy, np.float64)
        do.append((dy @ w).reshape(o.shape))
        dw += dy.T @ np.asarray(o, np.float64).reshape(n, -1)
    return do, dw
