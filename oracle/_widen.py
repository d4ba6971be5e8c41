"""Exact widening of the stored input formats to float64 (oracle-private)."""
import numpy as np


def bf16(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64, exactly."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def f32(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float32).astype(np.float64)
