"""Pins for the oracle's per-group quantiser (cold-page tiers).

Checked against brute force (argmin over every code with exact rational arithmetic),
hand-derived fixtures, closed forms and the round-trip error bound.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle.fp import fp16_rne_sat
from oracle.quant import (GROUP, TIER_I1, TIER_I2, TIER_I4, TIER_I8, dequant_int, quantise_int,
                          quantise_sign, quantise_token)

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _half_groups(rng, n, scale=1.0, dtype="f16"):
    x = rng.standard_normal((n, GROUP)) * scale
    if dtype == "f16":
        return x.astype(np.float16).astype(np.float64)
    u = x.astype(np.float32).view(np.uint32).astype(np.uint64)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_codes_are_bruteforce_argmin(bits, dtype):
    """Each code is the argmin over all 2^b codes of |x - (zero + c*scale)|, ties to even c."""
    rng = np.random.default_rng(bits)
    x = _half_groups(rng, 60, scale=3.0, dtype=dtype)
    codes, scale, zero, *_ = quantise_int(x, bits)
    qmax = (1 << bits) - 1
    for i in range(x.shape[0]):
        s, z = Fraction(float(scale[i])), Fraction(float(zero[i]))
        for j in range(GROUP):
            if s == 0:
                assert codes[i, j] == 0
                continue
            xv = Fraction(float(x[i, j]))
            errs = [abs(xv - (z + c * s)) for c in range(qmax + 1)]
            best = min(errs)
            cands = [c for c in range(qmax + 1) if errs[c] == best]
            want = cands[0] if len(cands) == 1 else [c for c in cands if c % 2 == 0][0]
            assert codes[i, j] == want, (i, j)


def test_scale_zero_definitions():
    rng = np.random.default_rng(7)
    x = _half_groups(rng, 50, 2.0)
    for bits in (2, 4, 8):
        _, scale, zero, sb, zb, _ = quantise_int(x, bits)
        lo, hi = x.min(1), x.max(1)
        assert np.array_equal(zero, lo.astype(np.float16).astype(np.float64))
        assert np.array_equal(scale, ((hi - lo) / ((1 << bits) - 1)).astype(np.float16).astype(np.float64))
        assert np.array_equal(sb.view(np.float16).astype(np.float64), scale)
        assert np.array_equal(zb.view(np.float16).astype(np.float64), zero)


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_grid_exact_roundtrip(bits):
    """Values on the code grid (containing both ends) come back exactly."""
    qmax = (1 << bits) - 1
    rng = np.random.default_rng(11)
    for trial in range(20):
        s = 2.0 ** int(rng.integers(-6, 0))
        z = s * int(rng.integers(-64, 64))
        c = rng.integers(0, qmax + 1, GROUP)
        c[0], c[1] = 0, qmax
        x = z + c * s
        assert np.all(x.astype(np.float16).astype(np.float64) == x)
        codes, scale, zero, *_ = quantise_int(x[None], bits)
        assert scale[0] == s and zero[0] == z
        assert np.array_equal(codes[0], c)
        assert np.array_equal(dequant_int(codes, scale, zero)[0], x)


def test_constant_group_is_exact():
    for v in (0.0, 1.5, -3.25, 1000.0):
        x = np.full((1, GROUP), v)
        for bits in (2, 4, 8):
            codes, scale, zero, *_ = quantise_int(x, bits)
            assert scale[0] == 0 and np.all(codes == 0)
            assert np.all(dequant_int(codes, scale, zero) == v)


def test_zero_extremes_are_positive_zero():
    """The signs of zeros do not change a group's bytes: a zero min gives zero = +0, and
    an all-zero group (any mix of +0 and -0) gives scale = +0 and zero = +0."""
    pos = np.abs(np.linspace(0.0, 3.0, GROUP))
    for order in (1, -1):
        x = pos.copy()
        x[0] = -0.0
        x[5] = 0.0
        x = x[::order][None]
        for bits in (2, 4, 8):
            *_, sb, zb, _ = quantise_int(x, bits)
            assert int(zb[0]) == 0x0000 and int(sb[0]) != 0
            want = quantise_int(np.abs(x), bits)
            assert np.array_equal(quantise_int(x, bits)[0], want[0])
    z = np.zeros((1, GROUP))
    z[0, ::3] = -0.0
    for bits in (2, 4, 8):
        *_, sb, zb, _ = quantise_int(z, bits)
        assert int(sb[0]) == 0 and int(zb[0]) == 0
        *_, sb, zb, _ = quantise_int(-np.zeros((1, GROUP)), bits)
        assert int(sb[0]) == 0 and int(zb[0]) == 0


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_roundtrip_bound(bits, dtype):
    """|x - xhat| <= scale/2 for unclamped codes (before the fp32 rounding); clamped end
    codes carry the extra slack of the fp16 rounding of lo and of the scale."""
    rng = np.random.default_rng(100 + bits)
    x = _half_groups(rng, 20000, 1.0, dtype)
    x[::7] *= 8.0                                  # outlier-heavy groups
    codes, scale, zero, *_ = quantise_int(x, bits)
    qmax = (1 << bits) - 1
    exact = codes * scale[:, None] + zero[:, None]          # exact in fp64
    xhat = dequant_int(codes, scale, zero)
    raw = (x - zero[:, None]) / np.where(scale == 0, 1, scale)[:, None]
    unclamped = (raw >= -0.5) & (raw <= qmax + 0.5) & (scale[:, None] > 0)
    err = np.abs(x - exact)
    assert np.all(err[unclamped] <= scale[:, None].repeat(GROUP, 1)[unclamped] / 2)
    lo = x.min(1)
    ulp_lo = np.abs(np.spacing(lo.astype(np.float16)).astype(np.float64))
    ulp_s = np.abs(np.spacing(scale.astype(np.float16)).astype(np.float64))
    slack = ulp_lo / 2 + qmax * ulp_s / 2
    bound = np.maximum(scale / 2, slack)[:, None] + np.abs(np.spacing(xhat.astype(np.float32))) / 2
    assert np.all(np.abs(x - xhat) <= bound)


def test_sign_tier_optimal_magnitude():
    """m = mean|x| minimises sum (x - m sign x)^2; one fp16 ulp either way never does better."""
    rng = np.random.default_rng(5)
    x = _half_groups(rng, 300, 2.0)
    x[0, 3] = -0.0
    bits, m, m_bits, _ = quantise_sign(x)
    assert bits[0, 3] == 1                                     # -0 -> +
    sgn = np.where(bits == 1, 1.0, -1.0)
    assert np.all((sgn > 0) == (x >= 0))
    assert np.array_equal(m, (np.abs(x).sum(1) / GROUP).astype(np.float16).astype(np.float64))

    def sse(a):
        return ((x - a[:, None] * sgn) ** 2).sum(1)
    base = sse(m)
    up = np.nextafter(m.astype(np.float16), np.float16(np.inf)).astype(np.float64)
    dn = np.nextafter(m.astype(np.float16), np.float16(0)).astype(np.float64)
    assert np.all(sse(up) >= base) and np.all(sse(dn) >= base)


def test_fp16_metadata_saturates():
    x = np.zeros((1, GROUP))
    x[0, 0], x[0, 1] = -1e6, 1e6
    *_, ov = quantise_int(x, 4)
    assert ov[0]
    _, scale, zero, *_ = quantise_int(x, 4)
    assert zero[0] == -65504.0 and scale[0] == 65504.0


def test_golden_quant_fixtures():
    """Hand-derived examples (values worked out by hand from the quantiser definition)."""
    with open(os.path.join(GOLD, "quant_examples.json")) as f:
        cases = json.load(f)["cases"]
    for case in cases:
        x = np.array(case["x"], dtype=np.float64)
        if case["bits"] == 1:
            bits, m, *_ = quantise_sign(x[None])
            assert list(bits[0]) == case["codes"]
            assert m[0] == case["m"]
        else:
            codes, scale, zero, *_ = quantise_int(x[None], case["bits"])
            assert list(codes[0]) == case["codes"], case["name"]
            assert scale[0] == case["scale"] and zero[0] == case["zero"], case["name"]


def test_quantise_token_meta_word():
    rng = np.random.default_rng(3)
    x = _half_groups(rng, 4).reshape(128)
    for tier in (TIER_I8, TIER_I4, TIER_I2):
        r = quantise_token(x, tier)
        meta = r["meta"]
        assert meta.shape == (4,)
        sc = (meta & 0xFFFF).astype(np.uint16).view(np.float16)
        ze = (meta >> 16).astype(np.uint16).view(np.float16)
        g = x.reshape(4, 32)
        assert np.array_equal(ze.astype(np.float64), fp16_rne_sat(g.min(1))[0])
        assert np.all(sc >= 0)
    r = quantise_token(x, TIER_I1)
    assert r["meta"].shape == (4,) and set(np.unique(r["codes"])) <= {0, 1}
