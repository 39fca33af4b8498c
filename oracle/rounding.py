"""Rounding of exact (fp64) values to the storage dtypes of the logits.

Test infrastructure only: part of the CPU oracle.

bfloat16 is the IEEE-754 binary32 layout cut to 7 fraction bits: 1 sign bit,
the 8-bit exponent of binary32 (normal range 2^-126 .. 2^127, subnormals down
to 2^-133) and an 8-bit significand. Rounding is round-to-nearest, ties to
even, the IEEE default. The function below rounds an fp64 value to it in ONE
step (no detour through fp32, which would round twice).
"""
from __future__ import annotations

import numpy as np

BF16_FRACTION_BITS = 7
BF16_MIN_NORMAL_EXP = -126
BF16_OVERFLOW = 2.0 ** 128  # first magnitude past the largest finite bfloat16


def round_to_bfloat16(x) -> np.ndarray:
    """Round fp64 values to the nearest bfloat16, ties to even; returns fp64
    holding bfloat16 values exactly. NaN stays NaN, +-inf stays +-inf, and a
    finite value that rounds past the largest finite bfloat16 becomes +-inf.
    """
    x = np.asarray(x, dtype=np.float64)
    out = x.copy()
    fin = np.isfinite(x)
    xf = x[fin]
    # xf = m * 2**e with 0.5 <= |m| < 1, so the binade of xf is 2**(e-1).
    _, e = np.frexp(xf)
    # Spacing of bfloat16 values in that binade (fixed at 2**-133 below the
    # normal range, where the format is subnormal).
    q = np.maximum(e - 1, BF16_MIN_NORMAL_EXP) - BF16_FRACTION_BITS
    scaled = np.ldexp(xf, -q)  # exact: a power-of-two scaling
    y = np.ldexp(np.rint(scaled), q)  # np.rint rounds half to even
    y = np.where(np.abs(y) >= BF16_OVERFLOW, np.copysign(np.inf, y), y)
    out[fin] = y
    return out


def round_to_float32(x) -> np.ndarray:
    """Round fp64 values to the nearest binary32 (numpy's cast, which is IEEE
    round-to-nearest-even), returned as fp64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def round_to(dtype: str, x) -> np.ndarray:
    if dtype == "bf16":
        return round_to_bfloat16(x)
    if dtype == "fp32":
        return round_to_float32(x)
    raise ValueError(f"unsupported logits dtype {dtype!r}")


def ulp_bfloat16(x) -> np.ndarray:
    """Spacing of bfloat16 values at |x| (the unit in the last place)."""
    x = np.abs(np.asarray(x, dtype=np.float64))
    _, e = np.frexp(np.where(x > 0, x, 1.0))
    q = np.maximum(e - 1, BF16_MIN_NORMAL_EXP) - BF16_FRACTION_BITS
    return np.ldexp(np.ones_like(x), q)
