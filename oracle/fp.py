"""Floating-point conversions used by the oracle (fp64 in, IEEE round-half-even out).

Test infrastructure only (see ``oracle/__init__.py``).
"""
from __future__ import annotations

import numpy as np

FP16_MAX = 65504.0


def f16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def bits16_to_f64(bits: np.ndarray, dtype: str) -> np.ndarray:
    """Exact value of 16-bit patterns of the cache dtype ('f16' or 'bf16')."""
    return f16_bits_to_f64(bits) if dtype == "f16" else bf16_bits_to_f64(bits)


def fp16_rne_sat(x: np.ndarray):
    """Round fp64 values to fp16 (round-half-even), saturating at +-65504.

    Returns ``(value_as_f64, bits_uint16, overflowed_mask)``.  Values whose rounding
    would give +-inf are saturated to +-65504 and reported in the mask.  numpy's
    float64 -> float16 conversion rounds once, directly from the double (pinned in
    ``tests/test_oracle_fp.py`` against exact rational rounding).
    """
    x = np.asarray(x, dtype=np.float64)
    with np.errstate(over="ignore", invalid="ignore"):
        h = x.astype(np.float16)
    over = np.isinf(h) & np.isfinite(x)
    h = np.where(over, np.copysign(np.float16(FP16_MAX), x).astype(np.float16), h)
    return h.astype(np.float64), h.view(np.uint16), over


def f32_rne(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to fp32 (round-half-even), returned as fp64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def two_sum_exact(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """True where the fp64 sum ``a + b`` is exact (Knuth's TwoSum error term is zero)."""
    s = a + b
    bb = s - a
    err = (a - (s - bb)) + (b - bb)
    return err == 0.0
