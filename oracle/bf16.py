"""Rounding of float64 values to bfloat16 and to float32 (oracle, test infrastructure).

bfloat16 keeps the float32 exponent range and 8 significant bits (7 stored).
Rounding is to nearest, ties to even, applied once, directly from float64
(no intermediate float32 rounding). The low-rank factors are held in 16 bits
(SVDQuant explainer, section 3: the low-rank branch is kept at 16-bit
precision); the encoder input is float32 (reading recorded in the design notes).
"""
import numpy as np


def round_bf16(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value (ties to even).

    Uses ``frexp``: ``x = m * 2**e`` with ``0.5 <= |m| < 1``; bf16 keeps 8
    significant bits, i.e. ``m`` on a grid of ``2**-8``. ``np.rint`` rounds
    half to even. Values below the bf16 normal range are not expected here
    and are rejected.
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    if np.any((x != 0) & (e < -125)):
        raise ValueError("subnormal bf16 results are outside the oracle's range")
    r = np.rint(m * 256.0) / 256.0
    return np.ldexp(r, e)


def round_f32(x) -> np.ndarray:
    """Round float64 values to float32 (IEEE round-to-nearest-even), returned as float64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def bf16_bits(x) -> np.ndarray:
    """uint16 bit patterns of values that are exactly bf16 (float64 input)."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32)
    if np.any(u & 0xFFFF):
        raise ValueError("value is not exactly representable in bf16")
    return (u >> 16).astype(np.uint16)


def from_bf16_bits(b) -> np.ndarray:
    """float64 values of uint16 bf16 bit patterns."""
    u = np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)
