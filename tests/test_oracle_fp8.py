"""Pins of the oracle's FP8 (e4m3) tier: the code table, round-half-even with
saturation, the per-group scale and the round-trip bound.

Checked against the e4m3 definition at hand-picked codes, torch's float8_e4m3fn decode
and conversion (an independent implementation), and brute force over all codes with
exact rational arithmetic.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle.layout import pack_chunk, unpack_chunk
from oracle.quant import (E4M3_MAX, GROUP, TIER_F8, dequant_fp8, e4m3_rne, e4m3_value, quantise_fp8,
                          quantise_token)


def test_hand_picked_codes():
    assert e4m3_value(0x7E) == 448.0 and e4m3_value(0xFE) == -448.0
    assert e4m3_value(0x38) == 1.0 and e4m3_value(0x40) == 2.0 and e4m3_value(0xB8) == -1.0
    assert e4m3_value(0x08) == 2.0 ** -6 and e4m3_value(0x01) == 2.0 ** -9 and e4m3_value(0x07) == 7 * 2.0 ** -9
    assert np.isnan(e4m3_value(0x7F)) and np.isnan(e4m3_value(0xFF))
    z = e4m3_value(0x80)
    assert z == 0.0 and np.signbit(z)


def test_table_matches_torch_decode():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = e4m3_value(codes)
    fin = np.isfinite(ref)
    assert np.array_equal(fin, np.isfinite(mine))
    assert np.array_equal(ref[fin], mine[fin])


def test_rounding_matches_torch_in_range_including_ties():
    rng = np.random.default_rng(0)
    grid = e4m3_value(np.arange(0x7F))
    mids = (grid[:-1] + grid[1:]) / 2                       # every tie, exact in fp32
    vals = np.concatenate([rng.uniform(-448, 448, 20000), rng.normal(0, 0.01, 5000), mids, -mids, grid, -grid,
                           [0.0, -0.0]]).astype(np.float32)
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy().astype(np.int64)
    assert np.array_equal(e4m3_rne(vals.astype(np.float64)), ref)


def test_rounding_is_nearest_with_ties_to_even_bruteforce():
    rng = np.random.default_rng(1)
    grid = [Fraction(float(v)) for v in e4m3_value(np.arange(0x7F))]
    for v in list(rng.uniform(0, 500, 400)) + [float(g) * 1.0000001 for g in e4m3_value(np.arange(0, 0x7F, 7))]:
        fv = Fraction(float(min(v, E4M3_MAX)))
        d = [abs(fv - g) for g in grid]
        best = min(d)
        cands = [i for i, x in enumerate(d) if x == best]
        want = cands[0] if len(cands) == 1 else [c for c in cands if c % 2 == 0][0]
        assert int(e4m3_rne(np.array(v))) == want, v


def test_saturation_and_signs():
    assert int(e4m3_rne(np.array(1e9))) == 0x7E and int(e4m3_rne(np.array(-470.0))) == 0xFE
    assert int(e4m3_rne(np.array(-0.0))) == 0x80 and int(e4m3_rne(np.array(-1e-9))) == 0x80
    assert int(e4m3_rne(np.array(np.nan))) == 0x7F


def test_group_scale_and_roundtrip_bound():
    rng = np.random.default_rng(2)
    x = rng.normal(0, 1, (500, GROUP)) * rng.uniform(1e-3, 100, (500, 1))
    x = x.astype(np.float32).astype(np.float64)
    codes, scale, sbits, ov = quantise_fp8(x)
    assert not ov.any()
    amax = np.abs(x).max(axis=1)
    assert np.allclose(scale, amax / 448.0, rtol=2.0 ** -11)
    q = x / scale[:, None]
    grid = e4m3_value(np.arange(0x7F))
    # the chosen value is the nearest grid point to the quotient: within half the local gap
    idx = np.clip(np.searchsorted(grid, np.minimum(np.abs(q), 448.0)), 1, 0x7E)
    gap = grid[idx] - grid[idx - 1]
    err = np.abs(np.abs(q) - np.abs(e4m3_value(codes)))
    assert np.all(err <= gap / 2 + 1e-12 + np.maximum(np.abs(q) - 448.0, 0))
    xhat = dequant_fp8(codes, scale)
    assert np.all(np.abs(x - xhat) <= scale[:, None] * (gap / 2 + 1e-9) + np.abs(x) * 2.0 ** -10)
    assert np.array_equal(xhat.astype(np.float32).astype(np.float64), xhat)   # exact in fp32


def test_zero_group_and_token_meta():
    z = np.zeros((1, GROUP))
    z[0, ::2] = -0.0
    codes, scale, sbits, _ = quantise_fp8(z)
    assert scale[0] == 0 and int(sbits[0]) == 0 and np.all(codes == 0)
    rng = np.random.default_rng(3)
    x = rng.normal(size=128).astype(np.float16).astype(np.float64)
    r = quantise_token(x, TIER_F8)
    assert r["meta"].shape == (4,) and np.all(r["meta"] < 0x10000)
    data = pack_chunk("k", TIER_F8, 128, 1, r["codes"][None], r["meta"][None])
    codes2, meta2 = unpack_chunk("k", TIER_F8, 128, data)
    assert np.array_equal(codes2[0], r["codes"]) and np.array_equal(meta2[0], r["meta"])


def test_hand_derived_fixture():
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "fp8_examples.json")) as f:
        fx = json.load(f)
    for e in fx["rounding"]:
        assert int(e4m3_rne(np.array(e["value"]))) == e["code"], e
    g = fx["group"]
    x = np.zeros(GROUP)
    x[:len(g["x"])] = g["x"]
    codes, scale, sbits, _ = quantise_fp8(x[None])
    assert int(sbits[0]) == g["scale_bits"]
    assert list(codes[0, :len(g["codes"])]) == g["codes"]


def test_nonfinite_group_reads_back_nan():
    """A group holding an infinite or NaN value (the library flags such input) stores the
    fp16 quiet NaN 0x7E00 as its scale and zero codes: every element reads back as NaN,
    whichever 16-bit type later consumes it.  Finite groups beside it are unchanged."""
    rng = np.random.default_rng(9)
    x = rng.normal(size=(4, GROUP)).astype(np.float16).astype(np.float64)
    ref_codes, ref_scale, ref_bits, _ = quantise_fp8(x)
    x[1, 5] = np.nan
    x[2, 0] = np.inf
    x[3, 31] = -np.inf
    codes, scale, sbits, _ = quantise_fp8(x)
    for i in (1, 2, 3):
        assert int(sbits[i]) == 0x7E00 and np.isnan(scale[i]) and np.all(codes[i] == 0)
        assert np.all(np.isnan(dequant_fp8(codes, scale)[i]))
    assert int(sbits[0]) == int(ref_bits[0]) and np.array_equal(codes[0], ref_codes[0])
    r = quantise_token(x.reshape(-1), TIER_F8)
    assert list(r["meta"]) == [int(ref_bits[0]), 0x7E00, 0x7E00, 0x7E00]
