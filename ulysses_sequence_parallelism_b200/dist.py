"""Ulysses across processes: one process per GPU, each holding ONE rank's
sequence shards, the two all-to-alls per layer done by a torch.distributed
process group (NCCL over NVLink/NVSwitch on B200 nodes).

Per layer (theaicatchup.com, "How Does Ulysses Sequence Parallelism Actually
Work?"): every rank holds N/P tokens of Q, K, V; an all-to-all gives each rank
the whole sequence for H/P query heads and H_kv/P key/value heads; attention
runs on those heads alone (they do not interact); a second all-to-all returns
each token's output to the rank that owns it. The Spanish note
(contenidos2-1ml.pages.dev, "¿Qué cambia en la práctica…?") wants NVLink for
this exchange so that it does not become the bottleneck; here it is split into
head chunks (whole GQA groups) so that the exchange of one chunk overlaps the
attention of the previous one.

Data path of one chunk c (heads [lo, lo + f) of every rank's H/P):
  ulysses_a2a_pack     sequence shard -> send [P][N/P][f][d]
  all_to_all_single    send -> recv, which IS the [N, f, d] head fragment
  ulysses_attn_fwd     P = 1, H = f on the fragment -> O fragment [N, f, d]
  all_to_all_single    O fragment (already [P][N/P][f][d]) -> recv_o
  ulysses_a2a_unpack   recv_o -> the chunk's head columns of the O shard
Backward: dO goes the same way in, dQ/dK/dV the same way out; the forward's
head fragments and LSE are kept for it.

Collectives are issued with ``async_op=True``: the process group runs them on
its own stream after the work already queued on the current stream, and
``wait()`` makes the current stream wait for them, so the kernels of chunk c
run while chunk c+1 is on the wire. Every rank issues the same collectives in
the same order.

``ExchangePlan`` holds the host-side schedule (chunks, buffer shapes, step
order). ``UlyssesDistLayer`` binds it to the library's CUDA kernels; its
``kernels`` argument exists so that tests can check the exchange choreography
on CPU process groups (gloo) with host implementations of the four kernel
steps. The default is the CUDA library, with no fallback: if the library is
missing every call raises.
"""
from typing import List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist

from . import api


class ExchangePlan:
    """Schedule of one layer's exchange over P processes.

    chunk_heads: query heads per rank in one chunk (a multiple of H/H_kv that
    divides H/P). Default: two chunks when the rank's heads hold at least two
    GQA groups in an even number (so one chunk's exchange can overlap the
    other's attention), else one chunk of all of them."""

    def __init__(self, N: int, P: int, H: int, H_kv: int, d: int, chunk_heads: Optional[int] = None):
        if P < 1 or N % P or H % P or H_kv % P or H % H_kv:
            raise ValueError("need N, H and H_kv divisible by P and H divisible by H_kv")
        self.N, self.P, self.H, self.H_kv, self.d = N, P, H, H_kv, d
        self.n = N // P
        self.g = H // H_kv
        self.hl = H // P
        groups = self.hl // self.g
        if chunk_heads is None:
            chunk_heads = self.hl // 2 if (groups >= 2 and groups % 2 == 0) else self.hl
        if chunk_heads < self.g or chunk_heads % self.g or self.hl % chunk_heads:
            raise ValueError(f"chunk_heads must be a multiple of H/H_kv = {self.g} dividing H/P = {self.hl}")
        self.f = chunk_heads
        self.fk = chunk_heads // self.g
        self.chunks: List[Tuple[int, int]] = [(lo, chunk_heads) for lo in range(0, self.hl, chunk_heads)]

    def send_shape(self, kv: bool) -> Tuple[int, int, int, int]:
        """[P, N/P, heads of the chunk, d] of one chunk's send/receive buffer."""
        return (self.P, self.n, self.fk if kv else self.f, self.d)

    def fragment_shape(self, kv: bool) -> Tuple[int, int, int]:
        """[N, heads of the chunk, d]: the same bytes as a receive buffer."""
        return (self.N, self.fk if kv else self.f, self.d)

    def forward_steps(self):
        """Order of the forward's steps: every chunk's inbound exchange is
        issued first (pack, all-to-all), then per chunk its attention, right
        after which its outbound all-to-all is issued, then the unpacks."""
        C = len(self.chunks)
        return ([(s, c) for c in range(C) for s in ("pack", "a2a_in")] + [("attn", c) for c in range(C)] +
                [("unpack", c) for c in range(C)])


class CudaKernels:
    """The library's kernels for the four local steps of the exchange."""

    @staticmethod
    def pack(plan, c, x0, x1, x2, s0, s1, s2):
        lo, f = plan.chunks[c]
        api.ulysses_a2a_pack(x0, x1, x2, s0, s1, s2, plan.N, plan.P, plan.H, plan.H_kv, plan.d, lo, f)

    @staticmethod
    def unpack(plan, c, r0, r1, r2, x0, x1, x2):
        lo, f = plan.chunks[c]
        api.ulysses_a2a_unpack(r0, r1, r2, x0, x1, x2, plan.N, plan.P, plan.H, plan.H_kv, plan.d, lo, f)

    @staticmethod
    def attn_fwd(plan, q, k, v, o, lse, cu_seqlens, scale):
        api.ulysses_attn_fwd([q], [k], [v], [o], [lse], plan.N, 1, plan.f, plan.fk, plan.d, cu_seqlens, 0, scale)

    @staticmethod
    def attn_bwd(plan, q, k, v, o, lse, do, dq, dk, dv, workspace, cu_seqlens, scale, deterministic):
        api.ulysses_attn_bwd([q], [k], [v], [o], [lse], [do], [dq], [dk], [dv], plan.N, 1, plan.f, plan.fk, plan.d,
                             workspace, cu_seqlens, 0, scale, deterministic=deterministic)

    @staticmethod
    def workspace_bytes(plan, deterministic):
        return api.ulysses_attn_bwd_workspace_size(plan.N, 1, plan.f, plan.fk, plan.d, deterministic)


class UlyssesDistLayer:
    """One Ulysses attention layer over the P processes of ``group``; this
    process holds rank ``dist.get_rank(group)``'s sequence shards
    ([N/P, H, d] for Q/O/dO/dQ, [N/P, H_kv, d] for K/V/dK/dV). Buffers are
    allocated once, so steps allocate nothing."""

    def __init__(self, N: int, H: int, H_kv: int, d: int, group=None, device=None, cu_seqlens=None,
                 softmax_scale: float = 0.0, chunk_heads: Optional[int] = None, backward: bool = True,
                 deterministic: bool = False, kernels=None):
        self.group = group
        P = dist.get_world_size(group)
        self.plan = ExchangePlan(N, P, H, H_kv, d, chunk_heads)
        self.k = kernels if kernels is not None else CudaKernels
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.cu = cu_seqlens
        self.scale = softmax_scale
        self.deterministic = deterministic
        self.backward_enabled = backward
        pl = self.plan
        bf = torch.bfloat16
        mk = lambda shape: torch.empty(shape, dtype=bf, device=self.device)
        C = len(pl.chunks)
        # inbound: send buffers, receive buffers (= head fragments, kept for the backward)
        self.send = [[mk(pl.send_shape(kv)) for kv in (False, True, True)] for _ in range(C)]
        self.frag = [[mk(pl.fragment_shape(kv)) for kv in (False, True, True)] for _ in range(C)]
        self.o_frag = [mk(pl.fragment_shape(False)) for _ in range(C)]
        self.lse = [torch.empty(pl.f, N, dtype=torch.float32, device=self.device) for _ in range(C)]
        self.recv_o = [mk(pl.send_shape(False)) for _ in range(C)]
        if backward:
            self.send_do = [mk(pl.send_shape(False)) for _ in range(C)]
            self.do_frag = [mk(pl.fragment_shape(False)) for _ in range(C)]
            self.dfrag = [[mk(pl.fragment_shape(kv)) for kv in (False, True, True)] for _ in range(C)]
            self.recv_d = [[mk(pl.send_shape(kv)) for kv in (False, True, True)] for _ in range(C)]
            self.workspace = torch.empty(max(1, self.k.workspace_bytes(pl, deterministic)), dtype=torch.uint8,
                                         device=self.device)

    def _a2a(self, out: torch.Tensor, inp: torch.Tensor):
        """Chunk q of ``inp`` (its leading P-way split) to rank q; ``out``
        receives rank p's chunk at position p. Asynchronous."""
        return dist.all_to_all_single(out.view(-1), inp.view(-1), group=self.group, async_op=True)

    def forward(self, q_seq: torch.Tensor, k_seq: torch.Tensor, v_seq: torch.Tensor,
                o_seq: Optional[torch.Tensor] = None) -> torch.Tensor:
        pl, K = self.plan, self.k
        if o_seq is None:
            o_seq = torch.empty_like(q_seq)
        works_in, works_out = {}, {}
        for step, c in pl.forward_steps():
            if step == "pack":
                s = self.send[c]
                K.pack(pl, c, q_seq, k_seq, v_seq, s[0], s[1], s[2])
            elif step == "a2a_in":
                works_in[c] = [self._a2a(self.frag[c][i], self.send[c][i]) for i in range(3)]
            elif step == "attn":
                for w in works_in.pop(c):
                    w.wait()
                f = self.frag[c]
                K.attn_fwd(pl, f[0], f[1], f[2], self.o_frag[c], self.lse[c], self.cu, self.scale)
                works_out[c] = [self._a2a(self.recv_o[c], self.o_frag[c])]   # outbound, right behind it
            elif step == "unpack":
                for w in works_out.pop(c):
                    w.wait()
                K.unpack(pl, c, self.recv_o[c], None, None, o_seq, None, None)
        return o_seq

    def backward(self, do_seq: torch.Tensor, dq_seq=None, dk_seq=None, dv_seq=None):
        if not self.backward_enabled:
            raise RuntimeError("layer built without backward buffers")
        pl, K = self.plan, self.k
        n = pl.n
        if dq_seq is None:
            dq_seq = torch.empty(n, pl.H, pl.d, dtype=torch.bfloat16, device=do_seq.device)
            dk_seq = torch.empty(n, pl.H_kv, pl.d, dtype=torch.bfloat16, device=do_seq.device)
            dv_seq = torch.empty(n, pl.H_kv, pl.d, dtype=torch.bfloat16, device=do_seq.device)
        C = len(pl.chunks)
        works_in = {}
        for c in range(C):
            K.pack(pl, c, do_seq, None, None, self.send_do[c], None, None)
            works_in[c] = self._a2a(self.do_frag[c], self.send_do[c])
        works_out = {}
        for c in range(C):
            works_in.pop(c).wait()
            f, g = self.frag[c], self.dfrag[c]
            K.attn_bwd(pl, f[0], f[1], f[2], self.o_frag[c], self.lse[c], self.do_frag[c], g[0], g[1], g[2],
                       self.workspace, self.cu, self.scale, self.deterministic)
            works_out[c] = [self._a2a(self.recv_d[c][i], g[i]) for i in range(3)]
        for c in range(C):
            for w in works_out.pop(c):
                w.wait()
            r = self.recv_d[c]
            K.unpack(pl, c, r[0], r[1], r[2], dq_seq, dk_seq, dv_seq)
        return dq_seq, dk_seq, dv_seq
