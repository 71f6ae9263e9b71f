"""The Ulysses attention layer as the pages' steps (test infrastructure only).

Per layer on every rank (theaicatchup.com, "How Does Ulysses Sequence
Parallelism Actually Work?"; radardeia.com, "Arquitetura Técnica"):
  1. each rank holds its chunk of N/P tokens (Q, K, V already projected);
  2. all-to-all: every rank ends up with all N positions for H/P heads;
  3. attention locally on those heads over the full sequence;
  4. reverse the shuffle: outputs return to sequence sharding.
The backward of an all-to-all is its inverse all-to-all (the pages train but
do not write the backward; this is the plainest reading), so dO is sent
seq -> head, attention backward runs per head, and dQ/dK/dV go head -> seq.
"""
from typing import List, Optional

import numpy as np

from .permute import seq_to_head, head_to_seq
from .attention import attention_forward, attention_backward


def ulysses_layer_forward(q_seq: List[np.ndarray], k_seq, v_seq, cu_seqlens=None,
                          scale: Optional[float] = None):
    """Sequence-sharded fp64 Q/K/V -> (sequence-sharded O, per-rank LSE [H/P, N])."""
    q_h, k_h, v_h = seq_to_head(q_seq), seq_to_head(k_seq), seq_to_head(v_seq)
    o_h, lse_h = [], []
    for r in range(len(q_seq)):
        o, lse = attention_forward(q_h[r], k_h[r], v_h[r], cu_seqlens, scale)
        o_h.append(o)
        lse_h.append(lse)
    return head_to_seq(o_h), lse_h


def ulysses_layer_backward(q_seq, k_seq, v_seq, do_seq, cu_seqlens=None,
                           scale: Optional[float] = None):
    """Sequence-sharded fp64 inputs and dO -> sequence-sharded (dQ, dK, dV)."""
    q_h, k_h, v_h = seq_to_head(q_seq), seq_to_head(k_seq), seq_to_head(v_seq)
    do_h = seq_to_head(do_seq)
    dq_h, dk_h, dv_h = [], [], []
    for r in range(len(q_seq)):
        dq, dk, dv = attention_backward(q_h[r], k_h[r], v_h[r], do_h[r], cu_seqlens, scale)
        dq_h.append(dq)
        dk_h.append(dk)
        dv_h.append(dv)
    return head_to_seq(dq_h), head_to_seq(dk_h), head_to_seq(dv_h)
