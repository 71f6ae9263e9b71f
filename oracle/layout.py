"""bf16 -> fp64 widening for the oracle (test infrastructure only).

A bf16 value is the upper 16 bits of an IEEE binary32; shifting the bit
pattern left by 16 gives that binary32 exactly, and binary32 -> binary64 is
exact, so the oracle sees exactly the values the GPU reads.
"""
import numpy as np


def widen_bf16(bits: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(bits).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)
