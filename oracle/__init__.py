"""CPU oracle for the Ulysses attention layer -- TEST INFRASTRUCTURE ONLY.

Plain, slow, fp64 numpy restatement of what one Ulysses attention layer
computes, written from the method's description (sequence sharding, an
all-to-all from sequence to head sharding, independent per-head causal
attention, the inverse all-to-all). Only ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline / reference arm may import it. The product
path (``ulysses_sequence_parallelism_b200``) never imports, calls or falls
back to anything here, and nothing here imports the product path.

Modules:
  layout     -- bf16 bit patterns -> fp64 (exact widening)
  permute    -- the two all-to-alls as index arithmetic (exact)
  attention  -- fp64 causal (varlen, GQA) softmax attention, forward and
                backward, straight from the definitions; sampled-row and
                sampled-column variants for the large workloads
  layer      -- the Ulysses layer as the pages' steps: a2a, attention, a2a
  brute      -- pure-Python triple-loop attention for tiny inputs (a pin)
  projection -- the QKV and output projections either side of the exchange

Every function pinned by tests in ``tests/test_oracle_pins.py``; there is no
unpinned function.
"""
from .layout import widen_bf16
from .permute import seq_to_head, head_to_seq
from .attention import (doc_starts, doc_ends, attention_forward, attention_backward,
                        bwd_preprocess, attention_rows, attention_kv_cols)
from .layer import ulysses_layer_forward, ulysses_layer_backward
from .projection import qkv_projection, out_projection, qkv_projection_backward, out_projection_backward

__all__ = ["widen_bf16", "seq_to_head", "head_to_seq", "doc_starts", "doc_ends",
           "attention_forward", "attention_backward", "bwd_preprocess",
           "attention_rows", "attention_kv_cols",
           "ulysses_layer_forward", "ulysses_layer_backward", "qkv_projection", "out_projection",
           "qkv_projection_backward", "out_projection_backward"]
