"""bf16 <-> float conversions for the oracle (test infrastructure only).

bf16 values arrive as uint16 bit patterns. Widening is exact: a bf16 value is an
fp32 value with the low 16 significand bits zero, and every fp32 value is an
fp64 value.
"""
import numpy as np


def widen(bits: np.ndarray) -> np.ndarray:
    """uint16 bf16 bits -> float64 (exact)."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def round_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float64 -> bf16 bits, round to nearest with ties to even, in one step.

    a = m * 2^e with 0.5 <= |m| < 1; a bf16 normal number keeps 8 significant
    bits, so the rounded value is rint(m * 2^8) * 2^(e-8) (``np.rint`` rounds
    half to even and m * 2^8 is exact). Below the smallest normal 2^-126 the
    grid is the fixed subnormal spacing 2^-133. Every result is exactly
    representable in fp32, so the final fp32 cast only reads off the bits.
    """
    a = np.asarray(a, dtype=np.float64)
    m, e = np.frexp(a)
    r = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)
    sub = np.abs(a) < 2.0 ** -126
    r = np.where(sub, np.ldexp(np.rint(np.ldexp(a, 133)), -133), r)
    return (r.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)
