"""Per-group quantisation of one token's head vector (the cold-page tiers).

Test infrastructure only (see ``oracle/__init__.py``).

ARGUS ("Virtual Memory for Transformers", sections "The One-Minute Explanation" and
"Visual Architecture") lists the tier cascade FP16 -> FP8 -> INT8 -> INT4 (two codes per
byte) -> INT2 (four per byte) -> 1-bit (eight signs per byte).  The pages do not fix the
quantiser, so this file takes the plainest affine reading and fixes every rounding:

* a group is 32 consecutive channels of one token of one head (K or V alike);
* ``lo`` and ``hi`` are the group's min and max as values: a zero extreme is +0 (the
  signs of the zeros in a group do not change its bytes);
* INT-b (b in {8, 4, 2}) is asymmetric min/max with a float zero offset:
  ``zero = fp16(lo)``, ``scale = fp16((hi - lo) / (2^b - 1))``,
  ``c = clamp(rint((x - zero) / scale), 0, 2^b - 1)`` (0 when scale == 0), and the
  value read back is ``fp32(c * scale + zero)`` with one rounding;
* 1-bit keeps the sign (``x >= 0`` -> +, so -0 -> +) and one magnitude per group,
  ``m = fp16(sum_j |x_j| / 32)`` (the L2-optimal alpha for ``alpha * sign(x)``), read
  back as ``+m`` or ``-m``;
* FP8 is e4m3 with one fp16 scale per group, ``scale = fp16(amax / 448)`` (448 the
  largest e4m3 value), ``code = e4m3(x / scale)`` rounded half to even with saturation,
  read back as ``e4m3(code) * scale``.

All intermediate steps are IEEE binary64 with round-half-even; fp16 results that
would overflow saturate to +-65504 and are reported.
"""
from __future__ import annotations

import numpy as np

from .fp import fp16_rne_sat, f32_rne, two_sum_exact

GROUP = 32
TIER_F16, TIER_I8, TIER_I4, TIER_I2, TIER_I1, TIER_F8 = 0, 1, 2, 3, 4, 5
TIER_BITS = {TIER_F16: 16, TIER_I8: 8, TIER_I4: 4, TIER_I2: 2, TIER_I1: 1, TIER_F8: 8}
E4M3_MAX = 448.0


def e4m3_value(code: np.ndarray) -> np.ndarray:
    """Value of an FP8 e4m3 code (OCP 8-bit float, 'fn' variant): sign, 4 exponent bits
    (bias 7), 3 mantissa bits; exponent 0 holds the subnormals m * 2^-9; 0x7F / 0xFF are
    NaN and there is no infinity (the largest finite value is 0x7E = 448)."""
    c = np.asarray(code, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * 2.0 ** (e.astype(np.float64) - 7.0))
    mag = np.where((c & 0x7F) == 0x7F, np.nan, mag)
    return sign * mag


def e4m3_rne(v: np.ndarray) -> np.ndarray:
    """Code of the e4m3 value nearest to ``v`` (fp64), ties to the even code, magnitudes
    beyond 448 saturating to 448, the sign of ``v`` kept (so -0 -> 0x80); NaN -> 0x7F."""
    v = np.asarray(v, dtype=np.float64)
    grid = e4m3_value(np.arange(0x7F))                    # the 127 finite magnitudes, ascending
    a = np.minimum(np.abs(v), E4M3_MAX)
    hi = np.searchsorted(grid, a, side="left")            # first grid value >= a
    hi = np.clip(hi, 0, 0x7E)
    lo = np.clip(hi - 1, 0, 0x7E)
    dlo, dhi = a - grid[lo], grid[hi] - a
    pick = np.where(dlo < dhi, lo, np.where(dhi < dlo, hi, np.where(lo % 2 == 0, lo, hi)))
    pick = np.where(a == grid[hi], hi, pick)
    code = pick | np.where(np.signbit(v), 0x80, 0)
    return np.where(np.isnan(v), 0x7F, code).astype(np.int64)


F8_NAN_SCALE_BITS = 0x7E00   # fp16 quiet NaN: the scale of a group holding a non-finite value


def quantise_fp8(x: np.ndarray):
    """FP8 tier of groups ``x[..., 32]``: ``scale = fp16(amax / 448)`` (amax the largest
    magnitude, a zero amax is +0), ``code = e4m3(x / scale)`` (fp64 quotient, then one
    round-half-even to e4m3 with saturation; all codes 0 when scale == 0); read back as
    ``e4m3(code) * scale`` (exact in fp32).  A group holding a non-finite value (flagged as
    such by the library) stores a NaN scale and zero codes, so every element reads back as
    NaN.  Returns ``(codes, scale, scale_bits, overflow)``."""
    x = np.asarray(x, dtype=np.float64)
    assert x.shape[-1] == GROUP
    bad = ~np.isfinite(x).all(axis=-1)
    amax = np.where(bad, 0.0, np.abs(np.where(np.isfinite(x), x, 0.0)).max(axis=-1)) + 0.0
    scale, scale_bits, ov = fp16_rne_sat(amax / E4M3_MAX)
    scale = np.where(bad, np.nan, scale)
    scale_bits = np.where(bad, F8_NAN_SCALE_BITS, scale_bits).astype(scale_bits.dtype)
    safe = np.where((scale == 0.0) | bad, 1.0, scale)
    codes = e4m3_rne(np.where(bad[..., None], 0.0, x) / safe[..., None])
    codes = np.where(((scale == 0.0) | bad)[..., None], 0, codes)
    return codes, scale, scale_bits, ov


def dequant_fp8(codes: np.ndarray, scale: np.ndarray) -> np.ndarray:
    return e4m3_value(codes) * scale[..., None]


def quantise_int(x: np.ndarray, bits: int):
    """Quantise groups ``x[..., 32]`` (fp64, exact cache values) to ``bits``-bit codes.

    Returns ``(codes int64 [..., 32], scale f64 [...], zero f64 [...],
    scale_bits u16, zero_bits u16, overflow bool [...])``.
    """
    x = np.asarray(x, dtype=np.float64)
    assert x.shape[-1] == GROUP
    qmax = float((1 << bits) - 1)
    lo = x.min(axis=-1) + 0.0   # a zero extreme is +0 whatever the signs of the zeros
    hi = x.max(axis=-1) + 0.0
    zero, zero_bits, ov0 = fp16_rne_sat(lo)
    scale, scale_bits, ov1 = fp16_rne_sat((hi - lo) / qmax)
    safe = np.where(scale == 0.0, 1.0, scale)
    c = np.rint((x - zero[..., None]) / safe[..., None])
    c = np.clip(c, 0.0, qmax)
    c = np.where((scale == 0.0)[..., None], 0.0, c)
    return c.astype(np.int64), scale, zero, scale_bits, zero_bits, ov0 | ov1


def dequant_int(codes: np.ndarray, scale: np.ndarray, zero: np.ndarray) -> np.ndarray:
    """``fp32(c * scale + zero)`` with a single rounding (returned as fp64).

    ``c * scale`` is exact in fp64 (8-bit code times 11-bit fp16 significand) and the
    sum with the fp16 zero is checked exact, so rounding the fp64 result to fp32 is
    the one rounding of a fused multiply-add.
    """
    codes = np.asarray(codes, dtype=np.float64)
    prod = codes * scale[..., None]
    zz = np.broadcast_to(zero[..., None], prod.shape)
    assert np.all(two_sum_exact(prod, zz)), "c*scale + zero is not exact in fp64"
    return f32_rne(prod + zz)


def quantise_sign(x: np.ndarray):
    """1-bit tier: sign bits and one fp16 magnitude per 32-channel group.

    The magnitude is the mean absolute value, summed sequentially over j = 0..31 in
    fp64 (exact for fp16 inputs; the fixed order makes it reproducible for bf16).
    Returns ``(bits int64 [..., 32] (1 = non-negative), m f64 [...], m_bits u16,
    overflow bool [...])``.
    """
    x = np.asarray(x, dtype=np.float64)
    assert x.shape[-1] == GROUP
    bits = (x >= 0.0).astype(np.int64)
    s = np.zeros(x.shape[:-1], dtype=np.float64)
    for j in range(GROUP):
        s = s + np.abs(x[..., j])
    m, m_bits, ov = fp16_rne_sat(s / GROUP)
    return bits, m, m_bits, ov


def dequant_sign(bits: np.ndarray, m: np.ndarray) -> np.ndarray:
    return np.where(np.asarray(bits) != 0, 1.0, -1.0) * m[..., None]


def quantise_token(x: np.ndarray, tier: int):
    """Quantise one token row ``x[D]`` (or rows ``x[..., D]``) into ``tier``.

    Returns a dict with ``codes [..., D]`` (int), ``meta`` (per group: for INT-b a
    uint32 ``scale_bits | zero_bits << 16``; for 1-bit the fp16 magnitude bits),
    ``xhat [..., D]`` (the value read back, fp64 holding an fp32) and ``overflow``.
    The 16-bit tier returns the input unchanged in ``xhat``.
    """
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    if tier == TIER_F16:
        return dict(codes=None, meta=None, xhat=x.copy(), overflow=np.zeros(x.shape[:-1], bool))
    g = x.reshape(*x.shape[:-1], D // GROUP, GROUP)
    if tier == TIER_F8:
        codes, scale, sbits, ov = quantise_fp8(g)
        return dict(codes=codes.reshape(x.shape), meta=sbits.astype(np.uint32),
                    xhat=dequant_fp8(codes, scale).reshape(x.shape), overflow=ov.any(axis=-1))
    if tier == TIER_I1:
        bits, m, m_bits, ov = quantise_sign(g)
        xhat = dequant_sign(bits, m)
        return dict(codes=bits.reshape(x.shape), meta=m_bits.astype(np.uint32),
                    xhat=xhat.reshape(x.shape), overflow=ov.any(axis=-1))
    b = TIER_BITS[tier]
    codes, scale, zero, sb, zb, ov = quantise_int(g, b)
    xhat = dequant_int(codes, scale, zero)
    meta = sb.astype(np.uint32) | (zb.astype(np.uint32) << 16)
    return dict(codes=codes.reshape(x.shape), meta=meta, xhat=xhat.reshape(x.shape),
                overflow=ov.any(axis=-1))
