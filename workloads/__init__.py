"""Seeded synthetic inputs for the Ulysses attention layer.

This module is shared by the CUDA path's tests/bench and by the CPU oracle.
It holds NO arithmetic of the method itself: it only names the workload
shapes, draws seeded random numbers, rounds them to bf16 once, and cuts the
unsharded token axis into the P contiguous sequence shards the method starts
from (each rank first takes one contiguous N/P-token piece of the sequence --
theaicatchup.com, "How Does Ulysses Sequence Parallelism Actually Work?").

Recipe (one numpy ``Generator(PCG64(seed))`` stream per workload, drawn in
this order): document lengths (packed-varlen workloads only), then Q, K, V,
then dO. Each tensor is drawn as float32 standard normals in token-major
``[N, heads, d]`` order, multiplied by the workload's ``scale`` and rounded to
bf16 with round-to-nearest-even. Values are returned as raw bf16 bit patterns
(``uint16``) so both consumers start from identical bytes.

Document lengths for packed workloads: ``L = floor(exp(U(ln lo, ln hi)))``,
drawn until the running total reaches N; the last document is cut to the
remainder.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "get", "draw_doc_lengths", "cu_seqlens_from_lengths",
    "round_to_bf16_bits", "generate", "seq_shards", "causal_pairs",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    N: int            # total tokens (all ranks)
    P: int            # sequence-parallel degree (virtual ranks)
    H: int            # query heads
    H_kv: int         # key/value heads (GQA)
    d: int            # head dim
    scale: float = 1.0          # multiplier on the N(0,1) draws
    backward: bool = True       # dO drawn, backward on the path
    varlen: Optional[tuple] = None   # (lo, hi) of the log-uniform doc lengths
    rank_sequential: bool = False    # virtual ranks processed one after another
    description: str = ""


WORKLOADS: Dict[str, Workload] = {
    w.name: w for w in [
        Workload("tiny", 512, 2, 8, 8, 64, backward=False,
                 description="N=512, P=2, H=H_kv=8, d=64, forward + inverse permute"),
        Workload("llama8k", 8192, 4, 32, 8, 128,
                 description="Llama-3-8B layer shape: N=8192, P=4, H=32, H_kv=8, d=128, fwd+bwd"),
        Workload("varlen64k", 65536, 4, 32, 8, 128, varlen=(1024, 16384),
                 description="packed varlen: N=65536, P=4, docs log-uniform in [1024,16384], fwd+bwd"),
        Workload("single64k", 65536, 4, 32, 8, 128,
                 description="64K single causal sequence (supplementary), fwd+bwd"),
        Workload("long96k", 98304, 4, 32, 8, 128, scale=0.5,
                 description="long single sequence: N=98304, P=4, 0.5*N(0,1), fwd+bwd"),
        Workload("million", 1048576, 8, 32, 8, 128, backward=False, rank_sequential=True,
                 description="million-token: N=1048576, P=8, fwd only, ranks one after another"),
    ]
}


def get(name: str) -> Workload:
    return WORKLOADS[name]


def draw_doc_lengths(rng: np.random.Generator, N: int, lo: int, hi: int) -> List[int]:
    """Log-uniform document lengths in [lo, hi] until they cover N tokens."""
    lengths: List[int] = []
    total = 0
    a, b = math.log(lo), math.log(hi)
    while total < N:
        L = int(math.floor(math.exp(rng.uniform(a, b))))
        L = min(L, N - total)
        lengths.append(L)
        total += L
    return lengths


def cu_seqlens_from_lengths(lengths) -> np.ndarray:
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return cu


def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def _draw_bf16(rng: np.random.Generator, shape, mult: float, chunk: int = 1 << 26) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        x = rng.standard_normal(e - s, dtype=np.float32)
        if mult != 1.0:
            x *= np.float32(mult)
        out[s:e] = round_to_bf16_bits(x)
    return out.reshape(shape)


def generate(w: Workload, seed: int = 0, N: Optional[int] = None, with_do: Optional[bool] = None):
    """Draw one workload's inputs. Returns a dict of uint16 bf16-bit arrays
    ``q [N,H,d]``, ``k``/``v`` ``[N,H_kv,d]``, optionally ``do [N,H,d]``, and
    ``cu_seqlens`` (int32, or None for a single causal sequence).

    ``N`` overrides the workload's token count (smaller parity cases drawn with
    the same recipe)."""
    N = w.N if N is None else N
    with_do = w.backward if with_do is None else with_do
    rng = np.random.Generator(np.random.PCG64(seed))
    cu = None
    if w.varlen is not None:
        cu = cu_seqlens_from_lengths(draw_doc_lengths(rng, N, *w.varlen))
    out = {"cu_seqlens": cu}
    out["q"] = _draw_bf16(rng, (N, w.H, w.d), w.scale)
    out["k"] = _draw_bf16(rng, (N, w.H_kv, w.d), w.scale)
    out["v"] = _draw_bf16(rng, (N, w.H_kv, w.d), w.scale)
    if with_do:
        out["do"] = _draw_bf16(rng, (N, w.H, w.d), 1.0)
    return out


def seq_shards(x: np.ndarray, P: int) -> List[np.ndarray]:
    """Rank p's sequence shard: tokens [p*N/P, (p+1)*N/P) (contiguous views)."""
    N = x.shape[0]
    assert N % P == 0
    n = N // P
    return [x[p * n:(p + 1) * n] for p in range(P)]


def causal_pairs(N: int, cu_seqlens=None) -> int:
    """Number of (i, j) pairs with j <= i inside one document: the unit that
    attention FLOPs are counted in."""
    if cu_seqlens is None:
        return N * (N + 1) // 2
    L = np.diff(np.asarray(cu_seqlens, dtype=np.int64))
    return int(np.sum(L * (L + 1) // 2))


def projection_inputs(N: int, H: int, H_kv: int, d: int, hidden: int, seed: int = 1):
    """Seeded synthetic hidden states and projection weights (bf16 bit
    patterns): x [N, hidden] ~ N(0, 1); W_qkv [(H + 2 H_kv) d, hidden] and
    W_o [hidden, H d] ~ N(0, 1/fan_in), so projected values stay O(1). One
    PCG64(seed) stream in the order x, W_qkv, W_o. No arithmetic of the method."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = _draw_bf16(rng, (N, hidden), 1.0)
    w_qkv = _draw_bf16(rng, ((H + 2 * H_kv) * d, hidden), 1.0 / math.sqrt(hidden))
    w_o = _draw_bf16(rng, (hidden, H * d), 1.0 / math.sqrt(H * d))
    return x, w_qkv, w_o
