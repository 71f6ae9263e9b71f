"""Helpers for the GPU parity tests: move bf16 bit patterns to/from the device
and compare against the fp64 oracle with the stated tolerances."""
import numpy as np
import torch

# Parity bar for bf16 attention outputs and gradients (O, dQ, dK, dV); see assert_close:
MAX_ABS = 2e-2
REL_RMS = 1e-2
# LSE is float32 end to end; its error comes from the fp32 online softmax and the
# approximate exp2/log2 (relative ~1e-6) on values of magnitude ln(N) + max score.
LSE_MAX_ABS = 2e-3


def to_dev(bits: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 bf16 bit patterns -> contiguous CUDA bf16 tensor (same bits)."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).to(device)


def bits_of(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def shards_to_dev(bits: np.ndarray, P: int):
    n = bits.shape[0] // P
    return [to_dev(bits[p * n:(p + 1) * n]) for p in range(P)]


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half the bf16 spacing at |x| (8 significant bits): the rounding error an
    exact result already carries once stored as bf16 with round-to-nearest-even."""
    ax = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, np.exp2(e - 8), 0.0)


def err_stats(gpu: np.ndarray, ref: np.ndarray):
    e = gpu - ref
    ma = float(np.max(np.abs(e))) if e.size else 0.0
    den = float(np.linalg.norm(ref))
    rr = float(np.linalg.norm(e) / den) if den > 0 else float(np.linalg.norm(e))
    return ma, rr


def assert_close(name, gpu, ref, max_abs=MAX_ABS, rel_rms=REL_RMS):
    """Parity bar for bf16 results: relative RMS error <= rel_rms, and max
    absolute error <= max_abs beyond the bf16 output's own half-ulp rounding
    (an exact result stored in bf16 is already up to 2^-6 off at |x| in [4, 8),
    2^-5 at [8, 16); the bar applies to the error the arithmetic adds)."""
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    ma, rr = err_stats(gpu, ref)
    excess = np.abs(gpu - ref) - bf16_half_ulp(ref)
    mx = float(np.max(excess)) if excess.size else 0.0
    if not (mx <= max_abs and rr <= rel_rms):
        i = np.unravel_index(int(np.argmax(excess)), excess.shape)
        big = int(np.sum(np.abs(ref) >= 4.0))
        raise AssertionError(
            f"{name}: max_abs {ma:.3e}, beyond half-ulp {mx:.3e} (<= {max_abs}), rel_rms {rr:.3e} (<= {rel_rms}); "
            f"worst at {i}: gpu {gpu[i]:.6f} ref {ref[i]:.6f}; {big} elements with |ref| >= 4")
    return ma, rr


def sample_rows(N: int, P: int, cu_seqlens, count: int, seed: int = 0, tile: int = 128):
    """Rows that stress the kernels: first/last token of every rank shard and of
    every document, tile edges (multiples of 128, +-1) and seeded uniform rows."""
    rng = np.random.Generator(np.random.PCG64(seed + 12345))
    n = N // P
    s = set()
    for p in range(P):
        s.update([p * n, p * n + n - 1])
    if cu_seqlens is not None:
        for c in np.asarray(cu_seqlens)[:-1]:
            s.update([int(c), min(N - 1, int(c) + 1)])
        for c in np.asarray(cu_seqlens)[1:]:
            s.add(int(c) - 1)
    edges = rng.choice(max(1, N // tile), size=min(count // 4, max(1, N // tile)), replace=False) * tile
    for e in edges:
        for x in (e - 1, e, e + 1):
            if 0 <= x < N:
                s.add(int(x))
    s.update(int(x) for x in rng.integers(0, N, size=count // 2))
    s.add(N - 1)
    rows = sorted(s)
    if len(rows) > count:
        keep = rng.choice(len(rows), size=count, replace=False)
        rows = sorted(rows[i] for i in keep) + [N - 1, 0]
    return sorted(set(rows))


def tail_cols(N: int, cu_seqlens, per_doc: int = 32):
    """Key positions at the end of each document (their gradients need only the
    few rows after them)."""
    ends = [N] if cu_seqlens is None else [int(x) for x in np.asarray(cu_seqlens)[1:]]
    starts = [0] if cu_seqlens is None else [int(x) for x in np.asarray(cu_seqlens)[:-1]]
    cols = []
    for a, b in zip(starts, ends):
        cols.extend(range(max(a, b - per_doc), b))
    return cols
