"""Thin Python binding over the C ABI (argument marshalling only).

Each function takes per-rank lists of CUDA tensors, checks dtype/device/
contiguity, passes raw device pointers plus the current CUDA stream to the
library, and raises ``UlyssesError`` on a non-zero status. Every step of the
layer runs in the library's kernels; PyTorch provides device memory and
streams. Shapes follow ``include/ulysses.h``:

  sequence shard of rank p : [N/P, Hx, d] bf16
  head shard of rank p     : [N, Hx/P, d] bf16
  LSE of rank p            : [H/P, N] float32
"""
import ctypes
from typing import List, Optional, Sequence

import torch

from ._lib import lib, check, UlyssesError, MAX_RANKS

__all__ = [
    "ulysses_a2a_seq_to_head", "ulysses_a2a_head_to_seq", "ulysses_attn_fwd", "ulysses_attn_bwd",
    "ulysses_attn_bwd_workspace_size", "ulysses_attn_bwd_seq_workspace_size", "ulysses_get_device_status",
    "ulysses_set_wait_limit",
    "ulysses_selftest_bounded_wait", "ulysses_attn_fwd_seq", "ulysses_attn_bwd_seq", "UlyssesLayer",
    "HostPipeline", "ulysses_a2a_seq_to_head_frag", "ulysses_a2a_head_to_seq_frag",
    "ulysses_qkv_proj_seq_to_head", "ulysses_out_proj_head_to_seq", "ulysses_out_proj_bwd",
    "ulysses_qkv_proj_bwd", "ulysses_a2a_pack", "ulysses_a2a_unpack",
]


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptrs(ts: Optional[Sequence[Optional[torch.Tensor]]], P: int, dtype=torch.bfloat16):
    if ts is None:
        return None
    if len(ts) != P:
        raise ValueError(f"expected {P} rank tensors, got {len(ts)}")
    arr = (ctypes.c_void_p * P)()
    for r, t in enumerate(ts):
        if t is None:
            arr[r] = None
            continue
        if not t.is_cuda or t.dtype != dtype or not t.is_contiguous():
            raise ValueError(f"rank {r}: need a contiguous CUDA {dtype} tensor, got {t.dtype} on {t.device}")
        arr[r] = t.data_ptr()
    return ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))


def _cu(cu_seqlens: Optional[torch.Tensor]):
    if cu_seqlens is None:
        return None, 0
    if not cu_seqlens.is_cuda or cu_seqlens.dtype != torch.int32:
        raise ValueError("cu_seqlens must be a CUDA int32 tensor")
    return ctypes.c_void_p(cu_seqlens.data_ptr()), cu_seqlens.numel() - 1


def ulysses_a2a_seq_to_head(x0_seq, x1_seq, x2_seq, x0_head, x1_head, x2_head, N, P, H, H_kv, d,
                            cu_seqlens=None, rank_lo=0, rank_hi=None, stream=None):
    cu, ns = _cu(cu_seqlens)
    code = lib().ulysses_a2a_seq_to_head(
        _ptrs(x0_seq, P), _ptrs(x1_seq, P), _ptrs(x2_seq, P), _ptrs(x0_head, P), _ptrs(x1_head, P),
        _ptrs(x2_head, P), N, P, H, H_kv, d, cu, ns, rank_lo, P if rank_hi is None else rank_hi, _stream(stream))
    check("ulysses_a2a_seq_to_head", code)


def ulysses_a2a_head_to_seq(x0_head, x1_head, x2_head, x0_seq, x1_seq, x2_seq, N, P, H, H_kv, d,
                            cu_seqlens=None, rank_lo=0, rank_hi=None, stream=None):
    cu, ns = _cu(cu_seqlens)
    code = lib().ulysses_a2a_head_to_seq(
        _ptrs(x0_head, P), _ptrs(x1_head, P), _ptrs(x2_head, P), _ptrs(x0_seq, P), _ptrs(x1_seq, P),
        _ptrs(x2_seq, P), N, P, H, H_kv, d, cu, ns, rank_lo, P if rank_hi is None else rank_hi, _stream(stream))
    check("ulysses_a2a_head_to_seq", code)


def _one(t: Optional[torch.Tensor], dtype=torch.bfloat16):
    if t is None:
        return None
    if not t.is_cuda or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"need a contiguous CUDA {dtype} tensor, got {t.dtype} on {t.device}")
    return ctypes.c_void_p(t.data_ptr())


def ulysses_a2a_seq_to_head_frag(x0_seq, x1_seq, x2_seq, x0_frag, x1_frag, x2_frag, N, P, H, H_kv, d, head_lo,
                                 num_heads, stream=None):
    """Global query heads [head_lo, head_lo + num_heads) (and their kv heads)
    of every token, from the P sequence shards into one fragment buffer each."""
    code = lib().ulysses_a2a_seq_to_head_frag(
        _ptrs(x0_seq, P), _ptrs(x1_seq, P), _ptrs(x2_seq, P), _one(x0_frag), _one(x1_frag), _one(x2_frag),
        N, P, H, H_kv, d, head_lo, num_heads, _stream(stream))
    check("ulysses_a2a_seq_to_head_frag", code)


def ulysses_a2a_head_to_seq_frag(x0_frag, x1_frag, x2_frag, x0_seq, x1_seq, x2_seq, N, P, H, H_kv, d, head_lo,
                                 num_heads, stream=None):
    code = lib().ulysses_a2a_head_to_seq_frag(
        _one(x0_frag), _one(x1_frag), _one(x2_frag), _ptrs(x0_seq, P), _ptrs(x1_seq, P), _ptrs(x2_seq, P),
        N, P, H, H_kv, d, head_lo, num_heads, _stream(stream))
    check("ulysses_a2a_head_to_seq_frag", code)


def ulysses_a2a_pack(x0_seq, x1_seq, x2_seq, x0_send, x1_send, x2_send, N, P, H, H_kv, d, head_lo=0,
                     num_heads=None, stream=None):
    """One rank's sequence shards -> per-destination chunks [P, N/P, f, d] of
    the head chunk [head_lo, head_lo + f) of every rank (for an all-to-all
    between processes)."""
    code = lib().ulysses_a2a_pack(
        _one(x0_seq), _one(x1_seq), _one(x2_seq), _one(x0_send), _one(x1_send), _one(x2_send), N, P, H, H_kv, d,
        head_lo, H // P if num_heads is None else num_heads, _stream(stream))
    check("ulysses_a2a_pack", code)


def ulysses_a2a_unpack(x0_recv, x1_recv, x2_recv, x0_seq, x1_seq, x2_seq, N, P, H, H_kv, d, head_lo=0,
                       num_heads=None, stream=None):
    """Inverse of ulysses_a2a_pack: received chunks [P, N/P, f, d] -> the
    chunk's head columns of this rank's sequence shards."""
    code = lib().ulysses_a2a_unpack(
        _one(x0_recv), _one(x1_recv), _one(x2_recv), _one(x0_seq), _one(x1_seq), _one(x2_seq), N, P, H, H_kv, d,
        head_lo, H // P if num_heads is None else num_heads, _stream(stream))
    check("ulysses_a2a_unpack", code)


def ulysses_qkv_proj_seq_to_head(x_seq, w_qkv, q_head, k_head, v_head, N, P, H, H_kv, d, hidden, stream=None):
    """[Q|K|V] = X W_qkv^T for every token, stored straight into the head shards."""
    code = lib().ulysses_qkv_proj_seq_to_head(
        _ptrs(x_seq, P), _one(w_qkv), _ptrs(q_head, P), _ptrs(k_head, P), _ptrs(v_head, P), N, P, H, H_kv, d,
        hidden, _stream(stream))
    check("ulysses_qkv_proj_seq_to_head", code)


def ulysses_out_proj_head_to_seq(o_head, w_o, y_seq, N, P, H, H_kv, d, hidden, stream=None):
    """Y = O W_o^T for every token, O read straight from the head shards."""
    code = lib().ulysses_out_proj_head_to_seq(
        _ptrs(o_head, P), _one(w_o), _ptrs(y_seq, P), N, P, H, H_kv, d, hidden, _stream(stream))
    check("ulysses_out_proj_head_to_seq", code)


def ulysses_out_proj_bwd(o_head, w_o, dy_seq, do_head, dw_o, N, P, H, H_kv, d, hidden, stream=None):
    """dO = dY W_o into the head shards; dW_o (fp32) = sum_t dy_t^T o_t."""
    code = lib().ulysses_out_proj_bwd(
        _ptrs(o_head, P), _one(w_o), _ptrs(dy_seq, P), _ptrs(do_head, P), _one(dw_o, torch.float32), N, P, H,
        H_kv, d, hidden,
        _stream(stream))
    check("ulysses_out_proj_bwd", code)


def ulysses_qkv_proj_bwd(x_seq, w_qkv, dq_head, dk_head, dv_head, dx_seq, dw_qkv, N, P, H, H_kv, d, hidden,
                         stream=None):
    """dX = [dQ|dK|dV] W_qkv into the sequence shards; dW_qkv (fp32) = sum_t g_t^T x_t."""
    code = lib().ulysses_qkv_proj_bwd(
        _ptrs(x_seq, P), _one(w_qkv), _ptrs(dq_head, P), _ptrs(dk_head, P), _ptrs(dv_head, P), _ptrs(dx_seq, P),
        _one(dw_qkv, torch.float32), N, P, H, H_kv, d, hidden, _stream(stream))
    check("ulysses_qkv_proj_bwd", code)


def ulysses_attn_fwd(q_head, k_head, v_head, o_head, lse_head, N, P, H, H_kv, d, cu_seqlens=None,
                     max_seqlen=0, softmax_scale=0.0, causal=1, rank_lo=0, rank_hi=None, stream=None):
    cu, ns = _cu(cu_seqlens)
    code = lib().ulysses_attn_fwd(
        _ptrs(q_head, P), _ptrs(k_head, P), _ptrs(v_head, P), _ptrs(o_head, P), _ptrs(lse_head, P, torch.float32),
        N, P, H, H_kv, d, cu, ns, max_seqlen, float(softmax_scale), causal, rank_lo,
        P if rank_hi is None else rank_hi, _stream(stream))
    check("ulysses_attn_fwd", code)


def ulysses_attn_fwd_seq(q_seq, k_seq, v_seq, o_seq, lse_head, N, P, H, H_kv, d, cu_seqlens=None,
                         max_seqlen=0, softmax_scale=0.0, causal=1, rank_lo=0, rank_hi=None, stream=None):
    cu, ns = _cu(cu_seqlens)
    code = lib().ulysses_attn_fwd_seq(
        _ptrs(q_seq, P), _ptrs(k_seq, P), _ptrs(v_seq, P), _ptrs(o_seq, P), _ptrs(lse_head, P, torch.float32),
        N, P, H, H_kv, d, cu, ns, max_seqlen, float(softmax_scale), causal, rank_lo,
        P if rank_hi is None else rank_hi, _stream(stream))
    check("ulysses_attn_fwd_seq", code)


def ulysses_attn_bwd_seq(q_seq, k_seq, v_seq, o_seq, lse_head, do_seq, dq_seq, dk_seq, dv_seq, N, P, H, H_kv, d,
                         workspace: torch.Tensor, cu_seqlens=None, max_seqlen=0, softmax_scale=0.0, rank_lo=0,
                         rank_hi=None, stream=None, deterministic=False):
    cu, ns = _cu(cu_seqlens)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    code = lib().ulysses_attn_bwd_seq(
        _ptrs(q_seq, P), _ptrs(k_seq, P), _ptrs(v_seq, P), _ptrs(o_seq, P), _ptrs(lse_head, P, torch.float32),
        _ptrs(do_seq, P), _ptrs(dq_seq, P), _ptrs(dk_seq, P), _ptrs(dv_seq, P), N, P, H, H_kv, d, cu, ns,
        max_seqlen, float(softmax_scale), int(bool(deterministic)), ctypes.c_void_p(workspace.data_ptr()),
        workspace.numel() * workspace.element_size(), rank_lo, P if rank_hi is None else rank_hi, _stream(stream))
    check("ulysses_attn_bwd_seq", code)


def ulysses_attn_bwd_workspace_size(N, P, H, H_kv, d, deterministic=False) -> int:
    return int(lib().ulysses_attn_bwd_workspace_size(N, P, H, H_kv, d, int(bool(deterministic))))


def ulysses_attn_bwd_seq_workspace_size(N, P, H, H_kv, d, deterministic=False) -> int:
    return int(lib().ulysses_attn_bwd_seq_workspace_size(N, P, H, H_kv, d, int(bool(deterministic))))


def ulysses_attn_bwd(q_head, k_head, v_head, o_head, lse_head, do_head, dq_head, dk_head, dv_head, N, P, H,
                     H_kv, d, workspace: torch.Tensor, cu_seqlens=None, max_seqlen=0, softmax_scale=0.0,
                     rank_lo=0, rank_hi=None, stream=None, deterministic=False):
    """deterministic=False (d=128): one-pass backward, dQ summed in fp32 by L2
    reductions (run-to-run low-bit differences in dQ). True: two-pass,
    bit-reproducible. The workspace must be sized with the same setting."""
    cu, ns = _cu(cu_seqlens)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    code = lib().ulysses_attn_bwd(
        _ptrs(q_head, P), _ptrs(k_head, P), _ptrs(v_head, P), _ptrs(o_head, P), _ptrs(lse_head, P, torch.float32),
        _ptrs(do_head, P), _ptrs(dq_head, P), _ptrs(dk_head, P), _ptrs(dv_head, P), N, P, H, H_kv, d, cu, ns,
        max_seqlen, float(softmax_scale), int(bool(deterministic)), ctypes.c_void_p(workspace.data_ptr()),
        workspace.numel() * workspace.element_size(), rank_lo, P if rank_hi is None else rank_hi, _stream(stream))
    check("ulysses_attn_bwd", code)


def ulysses_get_device_status(stream=None):
    """Synchronises the stream, reads and clears the device error word.
    Returns (status_code, raw_word)."""
    w = ctypes.c_uint32(0)
    code = lib().ulysses_get_device_status(_stream(stream), ctypes.byref(w))
    return code, w.value


def ulysses_set_wait_limit(iters: int):
    lib().ulysses_set_wait_limit(int(iters))


def ulysses_selftest_bounded_wait(stream=None):
    check("ulysses_selftest_bounded_wait", lib().ulysses_selftest_bounded_wait(_stream(stream)))


class UlyssesLayer:
    """One Ulysses attention layer over P virtual ranks of one GPU.

    Holds the head-sharded buffers (and the backward workspace) so repeated
    steps allocate nothing. ``forward`` runs seq->head (Q, K, V in one launch),
    attention forward, head->seq (O); ``backward`` runs seq->head (dO),
    attention backward, head->seq (dQ, dK, dV in one launch)."""

    def __init__(self, N: int, P: int, H: int, H_kv: int, d: int, device="cuda", cu_seqlens=None,
                 max_seqlen: int = 0, softmax_scale: float = 0.0, backward: bool = True,
                 rank_sequential: bool = False, fused: bool = False, deterministic: bool = False,
                 head_fragment: int = 0):
        if P > MAX_RANKS:
            raise ValueError(f"P <= {MAX_RANKS}")
        self.N, self.P, self.H, self.H_kv, self.d = N, P, H, H_kv, d
        self.cu = cu_seqlens
        self.max_seqlen = max_seqlen
        self.scale = softmax_scale
        self.rank_sequential = rank_sequential
        # deterministic: two-pass backward with bit-reproducible dQ (else one pass)
        self.deterministic = deterministic
        # fused: the all-to-alls happen inside the attention kernels' addressing
        # (ulysses_attn_fwd_seq / ulysses_attn_bwd_seq); no head-sharded copies.
        self.fused = fused
        if fused and (rank_sequential or (N // P) % 128 != 0):
            raise ValueError("the fused layer needs all ranks at once and N/P a multiple of 128")
        # head_fragment = f > 0: every rank processes its heads f at a time (whole GQA
        # groups), one fragment after another; only one fragment's full-sequence
        # buffers exist (ulysses_a2a_*_frag + attention with P = 1 on the fragment).
        self.frag = int(head_fragment)
        g = H // H_kv
        if self.frag:
            if fused or rank_sequential:
                raise ValueError("head_fragment excludes fused and rank_sequential")
            if self.frag % g != 0 or (H // P) % self.frag != 0:
                raise ValueError(f"head_fragment must be a multiple of H/H_kv = {g} dividing H/P = {H // P}")
        bf, f32 = torch.bfloat16, torch.float32
        nb = 1 if rank_sequential else P      # rank-sequential: one rank's head buffers, reused
        if fused or self.frag:
            nb = 0
        mk = lambda hx: [torch.empty(N, hx // P, d, dtype=bf, device=device) for _ in range(nb)]
        self.q_h, self.k_h, self.v_h, self.o_h = mk(H), mk(H_kv), mk(H_kv), mk(H)
        # LSE of every rank is kept (it is what a backward needs; [H/P, N] fp32 per
        # rank is small next to the head shards), also when ranks run one by one.
        self.lse = [torch.empty(H // P, N, dtype=f32, device=device) for _ in range(P)]
        self.backward_enabled = backward and not rank_sequential
        if self.frag:
            f, fk = self.frag, self.frag // g
            fb = lambda hx: torch.empty(N, hx, d, dtype=bf, device=device)
            self.q_f, self.k_f, self.v_f, self.o_f = fb(f), fb(fk), fb(fk), fb(f)
            if self.backward_enabled:
                self.do_f, self.dq_f, self.dk_f, self.dv_f = fb(f), fb(f), fb(fk), fb(fk)
                ws = ulysses_attn_bwd_workspace_size(N, 1, f, fk, d, deterministic)
                self.workspace = torch.empty(ws, dtype=torch.uint8, device=device)
        elif self.backward_enabled:
            self.do_h, self.dq_h, self.dk_h, self.dv_h = mk(H), mk(H), mk(H_kv), mk(H_kv)
            # fused: room for the backward to stage Q and dO in head shards
            size = ulysses_attn_bwd_seq_workspace_size if fused else ulysses_attn_bwd_workspace_size
            ws = size(N, P, H, H_kv, d, deterministic)
            self.workspace = torch.empty(ws, dtype=torch.uint8, device=device)

    def forward_projected(self, x_seq: List[torch.Tensor], w_qkv: torch.Tensor, w_o: torch.Tensor,
                          y_seq: Optional[List[torch.Tensor]] = None):
        """The attention block forward with its projections: hidden states
        x_seq[p] [N/P, hidden] -> y_seq[p] [N/P, hidden]. The QKV projection
        stores Q/K/V straight into the head shards and the output projection
        reads O straight from them, so neither all-to-all runs as a permute."""
        if self.fused or self.frag or self.rank_sequential:
            raise ValueError("forward_projected runs on the plain all-ranks layer")
        N, P, H, H_kv, d = self.N, self.P, self.H, self.H_kv, self.d
        hidden = x_seq[0].shape[1]
        if y_seq is None:
            y_seq = [torch.empty_like(x) for x in x_seq]
        ulysses_qkv_proj_seq_to_head(x_seq, w_qkv, self.q_h, self.k_h, self.v_h, N, P, H, H_kv, d, hidden)
        ulysses_attn_fwd(self.q_h, self.k_h, self.v_h, self.o_h, self.lse, N, P, H, H_kv, d, self.cu,
                         self.max_seqlen, self.scale)
        ulysses_out_proj_head_to_seq(self.o_h, w_o, y_seq, N, P, H, H_kv, d, hidden)
        return y_seq

    def backward_projected(self, dy_seq: List[torch.Tensor], x_seq: List[torch.Tensor], w_qkv: torch.Tensor,
                           w_o: torch.Tensor):
        """Backward of forward_projected (call it after forward_projected on the
        same layer): dY -> (dX sequence shards, dW_qkv, dW_o); weight
        gradients in fp32. dO goes straight
        into the head shards and dX is gathered straight from the attention
        gradients' head shards: no permute runs."""
        if not self.backward_enabled or self.fused or self.frag or self.rank_sequential:
            raise ValueError("backward_projected runs on the plain all-ranks layer with backward buffers")
        N, P, H, H_kv, d = self.N, self.P, self.H, self.H_kv, self.d
        hidden = x_seq[0].shape[1]
        dw_o = torch.empty(w_o.shape, dtype=torch.float32, device=w_o.device)
        dw_qkv = torch.empty(w_qkv.shape, dtype=torch.float32, device=w_qkv.device)
        dx_seq = [torch.empty_like(x) for x in x_seq]
        ulysses_out_proj_bwd(self.o_h, w_o, dy_seq, self.do_h, dw_o, N, P, H, H_kv, d, hidden)
        ulysses_attn_bwd(self.q_h, self.k_h, self.v_h, self.o_h, self.lse, self.do_h, self.dq_h, self.dk_h,
                         self.dv_h, N, P, H, H_kv, d, self.workspace, self.cu, self.max_seqlen, self.scale,
                         deterministic=self.deterministic)
        ulysses_qkv_proj_bwd(x_seq, w_qkv, self.dq_h, self.dk_h, self.dv_h, dx_seq, dw_qkv, N, P, H, H_kv, d, hidden)
        return dx_seq, dw_qkv, dw_o

    def _fragments(self):
        """(rank, head offset within the rank, global first query head) of every fragment."""
        hl = self.H // self.P
        for r in range(self.P):
            for j0 in range(0, hl, self.frag):
                yield r, j0, r * hl + j0

    def _rank_bufs(self, bufs, r):
        lst = [None] * self.P
        lst[r] = bufs[0]
        return lst

    def forward(self, q_seq: List[torch.Tensor], k_seq, v_seq, o_seq: Optional[List[torch.Tensor]] = None):
        N, P, H, H_kv, d = self.N, self.P, self.H, self.H_kv, self.d
        if o_seq is None:
            o_seq = [torch.empty_like(x) for x in q_seq]
        if self.fused:
            self._seq_in = (q_seq, k_seq, v_seq, o_seq)
            ulysses_attn_fwd_seq(q_seq, k_seq, v_seq, o_seq, self.lse, N, P, H, H_kv, d, self.cu, self.max_seqlen,
                                 self.scale)
        elif self.frag:
            self._seq_in = (q_seq, k_seq, v_seq, o_seq)
            f, fk = self.frag, self.frag // (H // H_kv)
            for r, j0, h_lo in self._fragments():
                ulysses_a2a_seq_to_head_frag(q_seq, k_seq, v_seq, self.q_f, self.k_f, self.v_f, N, P, H, H_kv, d,
                                             h_lo, f)
                ulysses_attn_fwd([self.q_f], [self.k_f], [self.v_f], [self.o_f], [self.lse[r][j0:j0 + f]], N, 1, f,
                                 fk, d, self.cu, self.max_seqlen, self.scale)
                ulysses_a2a_head_to_seq_frag(self.o_f, None, None, o_seq, None, None, N, P, H, H_kv, d, h_lo, f)
        elif not self.rank_sequential:
            ulysses_a2a_seq_to_head(q_seq, k_seq, v_seq, self.q_h, self.k_h, self.v_h, N, P, H, H_kv, d, self.cu)
            ulysses_attn_fwd(self.q_h, self.k_h, self.v_h, self.o_h, self.lse, N, P, H, H_kv, d, self.cu,
                             self.max_seqlen, self.scale)
            ulysses_a2a_head_to_seq(self.o_h, None, None, o_seq, None, None, N, P, H, H_kv, d, self.cu)
        else:
            for r in range(P):
                rb = lambda b: self._rank_bufs(b, r)
                ulysses_a2a_seq_to_head(q_seq, k_seq, v_seq, rb(self.q_h), rb(self.k_h), rb(self.v_h), N, P, H,
                                        H_kv, d, self.cu, rank_lo=r, rank_hi=r + 1)
                ulysses_attn_fwd(rb(self.q_h), rb(self.k_h), rb(self.v_h), rb(self.o_h), self.lse, N, P, H,
                                 H_kv, d, self.cu, self.max_seqlen, self.scale, rank_lo=r, rank_hi=r + 1)
                ulysses_a2a_head_to_seq(rb(self.o_h), None, None, o_seq, None, None, N, P, H, H_kv, d, self.cu,
                                        rank_lo=r, rank_hi=r + 1)
        return o_seq

    def backward(self, do_seq: List[torch.Tensor], dq_seq=None, dk_seq=None, dv_seq=None):
        if not self.backward_enabled:
            raise RuntimeError("layer built without backward buffers")
        N, P, H, H_kv, d = self.N, self.P, self.H, self.H_kv, self.d
        if dq_seq is None:
            dq_seq = [torch.empty(N // P, H, d, dtype=torch.bfloat16, device=do_seq[0].device) for _ in range(P)]
            dk_seq = [torch.empty(N // P, H_kv, d, dtype=torch.bfloat16, device=do_seq[0].device) for _ in range(P)]
            dv_seq = [torch.empty(N // P, H_kv, d, dtype=torch.bfloat16, device=do_seq[0].device) for _ in range(P)]
        if self.frag:
            q_seq, k_seq, v_seq, o_seq = self._seq_in
            f, fk = self.frag, self.frag // (H // H_kv)
            for r, j0, h_lo in self._fragments():
                ulysses_a2a_seq_to_head_frag(q_seq, k_seq, v_seq, self.q_f, self.k_f, self.v_f, N, P, H, H_kv, d,
                                             h_lo, f)
                ulysses_a2a_seq_to_head_frag(o_seq, None, None, self.o_f, None, None, N, P, H, H_kv, d, h_lo, f)
                ulysses_a2a_seq_to_head_frag(do_seq, None, None, self.do_f, None, None, N, P, H, H_kv, d, h_lo, f)
                ulysses_attn_bwd([self.q_f], [self.k_f], [self.v_f], [self.o_f], [self.lse[r][j0:j0 + f]],
                                 [self.do_f], [self.dq_f], [self.dk_f], [self.dv_f], N, 1, f, fk, d, self.workspace,
                                 self.cu, self.max_seqlen, self.scale, deterministic=self.deterministic)
                ulysses_a2a_head_to_seq_frag(self.dq_f, self.dk_f, self.dv_f, dq_seq, dk_seq, dv_seq, N, P, H, H_kv,
                                             d, h_lo, f)
            return dq_seq, dk_seq, dv_seq
        if self.fused:
            q_seq, k_seq, v_seq, o_seq = self._seq_in
            ulysses_attn_bwd_seq(q_seq, k_seq, v_seq, o_seq, self.lse, do_seq, dq_seq, dk_seq, dv_seq, N, P, H,
                                 H_kv, d, self.workspace, self.cu, self.max_seqlen, self.scale,
                                 deterministic=self.deterministic)
            return dq_seq, dk_seq, dv_seq
        ulysses_a2a_seq_to_head(do_seq, None, None, self.do_h, None, None, N, P, H, H_kv, d, self.cu)
        ulysses_attn_bwd(self.q_h, self.k_h, self.v_h, self.o_h, self.lse, self.do_h, self.dq_h, self.dk_h,
                         self.dv_h, N, P, H, H_kv, d, self.workspace, self.cu, self.max_seqlen, self.scale,
                         deterministic=self.deterministic)
        ulysses_a2a_head_to_seq(self.dq_h, self.dk_h, self.dv_h, dq_seq, dk_seq, dv_seq, N, P, H, H_kv, d, self.cu)
        return dq_seq, dk_seq, dv_seq


class HostPipeline:
    """Layer steps whose inputs and results live in host memory, through the
    C-ABI host pipeline (``ulysses_host_pipeline_*``; this class only
    marshals arguments and owns the device scratch buffer).

    ``submit(host_in, host_out)`` enqueues one step of ``layer``'s shape and
    options (forward + backward when the layer has backward buffers): the
    host->device copies of the step's sequence shards (Q, K, V, dO), the
    layer's kernels, and the device->host copies of its results (O, dQ, dK,
    dV). Copies in, compute and copies out run on three streams of the library
    with two device buffer sets, so the copies of neighbouring steps overlap
    this step's kernels and PCIe carries both directions at once. Results of a
    step are in ``host_out`` once ``synchronize()`` returns (or once the
    ``after`` event given to ``submit`` has completed).

    host_in:  {"q": [P tensors], "k": [...], "v": [...], "do": [...]}
    host_out: {"o": [...], "dq": [...], "dk": [...], "dv": [...]}
    (pinned CPU bf16 tensors shaped like the sequence shards; "do", "dq",
    "dk", "dv" only with backward). The layer's own device buffers are not
    used: the pipeline has its own in its scratch buffer.
    """

    def __init__(self, layer: "UlyssesLayer", device="cuda"):
        self.layer = layer
        self.bwd = bool(layer.backward_enabled)
        N, P, H, H_kv, d = layer.N, layer.P, layer.H, layer.H_kv, layer.d
        det = int(bool(layer.deterministic))
        nbytes = int(lib().ulysses_host_pipeline_scratch_bytes(N, P, H, H_kv, d, int(self.bwd), det))
        if nbytes == 0:
            raise UlyssesError("ulysses_host_pipeline_scratch_bytes", 2)
        self.scratch = torch.empty(nbytes, dtype=torch.uint8, device=device)
        handle = ctypes.c_void_p()
        check("ulysses_host_pipeline_create",
              lib().ulysses_host_pipeline_create(N, P, H, H_kv, d, int(self.bwd), det,
                                                 ctypes.c_void_p(self.scratch.data_ptr()), nbytes,
                                                 ctypes.byref(handle)))
        self.handle = handle
        self._cu, self._ns = _cu(layer.cu)

    @staticmethod
    def _host_ptrs(ts, P):
        if ts is None:
            return None
        if len(ts) != P:
            raise ValueError(f"expected {P} host shards, got {len(ts)}")
        arr = (ctypes.c_void_p * P)()
        for r, t in enumerate(ts):
            if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
                raise ValueError(f"rank {r}: need a contiguous host bf16 tensor")
            arr[r] = t.data_ptr()
        return ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))

    @staticmethod
    def _event(ev):
        if ev is None:
            return None
        if ev.cuda_event == 0:          # torch creates the event at its first record
            ev.record()
        return ctypes.c_void_p(ev.cuda_event)

    def submit(self, host_in, host_out, before=None, after=None):
        """before / after: optional torch.cuda.Event, recorded on the copy-in
        stream before the step's first copy and on the copy-out stream after
        its last."""
        P = self.layer.P
        used = ("q", "k", "v", "o") + (("do", "dq", "dk", "dv") if self.bwd else ())
        hp = lambda dct, key: self._host_ptrs(dct.get(key), P) if key in used else None
        check("ulysses_host_pipeline_submit",
              lib().ulysses_host_pipeline_submit(self.handle, hp(host_in, "q"), hp(host_in, "k"), hp(host_in, "v"),
                                                 hp(host_in, "do"), hp(host_out, "o"), hp(host_out, "dq"),
                                                 hp(host_out, "dk"), hp(host_out, "dv"), self._cu, self._ns,
                                                 float(self.layer.scale), self._event(before), self._event(after)))

    def synchronize(self):
        check("ulysses_host_pipeline_synchronize", lib().ulysses_host_pipeline_synchronize(self.handle))

    def close(self):
        if getattr(self, "handle", None) is not None and self.handle.value:
            lib().ulysses_host_pipeline_destroy(self.handle)
        self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
