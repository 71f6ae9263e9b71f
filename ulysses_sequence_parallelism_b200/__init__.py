"""Ulysses sequence-parallel attention layer for NVIDIA B200 (sm_100a).

The C ABI (``include/ulysses.h``) lives in ``libulysses_b200.so``, built
in-tree by ``build.py``; this package is a thin ctypes binding over it.
"""
from ._lib import UlyssesError, lib, LIB_PATH, exported_symbols
from .api import (ulysses_a2a_seq_to_head, ulysses_a2a_head_to_seq, ulysses_attn_fwd, ulysses_attn_bwd,
                  ulysses_attn_bwd_workspace_size, ulysses_attn_bwd_seq_workspace_size, ulysses_get_device_status, ulysses_set_wait_limit,
                  ulysses_selftest_bounded_wait, ulysses_attn_fwd_seq, ulysses_attn_bwd_seq,
                  UlyssesLayer, HostPipeline, ulysses_a2a_seq_to_head_frag, ulysses_a2a_head_to_seq_frag,
                  ulysses_qkv_proj_seq_to_head, ulysses_out_proj_head_to_seq, ulysses_out_proj_bwd,
                  ulysses_qkv_proj_bwd, ulysses_a2a_pack, ulysses_a2a_unpack)
from .dist import ExchangePlan, UlyssesDistLayer

__all__ = ["UlyssesError", "lib", "LIB_PATH", "exported_symbols", "ulysses_a2a_seq_to_head",
           "ulysses_a2a_head_to_seq", "ulysses_attn_fwd", "ulysses_attn_bwd", "ulysses_attn_bwd_workspace_size",
           "ulysses_attn_bwd_seq_workspace_size", "ulysses_get_device_status", "ulysses_set_wait_limit", "ulysses_selftest_bounded_wait", "ulysses_attn_fwd_seq",
           "ulysses_attn_bwd_seq", "UlyssesLayer", "HostPipeline",
           "ulysses_a2a_seq_to_head_frag", "ulysses_a2a_head_to_seq_frag", "ulysses_qkv_proj_seq_to_head",
           "ulysses_out_proj_head_to_seq", "ulysses_out_proj_bwd", "ulysses_qkv_proj_bwd", "ulysses_a2a_pack",
           "ulysses_a2a_unpack", "ExchangePlan", "UlyssesDistLayer"]
