"""Pins for the oracle's page byte layout: hand-derived positions, bijection, round trip."""
import json
import os

import numpy as np
import pytest

from oracle.layout import T, _positions, chunk_bytes, codes_bytes, pack_chunk, unpack_chunk
from oracle.quant import TIER_BITS

GOLD = os.path.join(os.path.dirname(__file__), "golden")
ALL = [(kind, tier, D) for kind in "kv" for tier in range(6) for D in (64, 128)]


def test_hand_derived_positions():
    with open(os.path.join(GOLD, "layout_examples.json")) as f:
        g = json.load(f)
    for e in g["positions"]:
        word, bit = _positions(e["kind"], e["tier"], e["D"])
        assert (int(word[e["t"], e["d"]]), int(bit[e["t"], e["d"]])) == (e["word"], e["bit"]), e


def test_hand_derived_i4_bytes():
    with open(os.path.join(GOLD, "layout_examples.json")) as f:
        ex = json.load(f)["i4_k_token0_codes_0_to_15"]["bytes"]
    codes = np.zeros((1, 128), dtype=np.int64)
    codes[0, :16] = np.arange(16)
    data = pack_chunk("k", 2, 128, 1, codes, np.zeros((1, 4), np.uint32))
    want = np.zeros(codes_bytes(2, 128), dtype=np.uint8)
    for off, v in ex.items():
        want[int(off)] = v
    assert np.array_equal(data[:codes_bytes(2, 128)], want)


@pytest.mark.parametrize("kind,tier,D", ALL)
def test_positions_are_a_bijection_onto_the_codes_area(kind, tier, D):
    b = TIER_BITS[tier]
    word, bit = _positions(kind, tier, D)
    nbits = codes_bytes(tier, D) * 8
    cover = np.zeros(nbits, dtype=np.int64)
    for w, s in zip(word.ravel(), bit.ravel()):
        assert s + b <= 32
        cover[w * 32 + s: w * 32 + s + b] += 1
    assert np.all(cover == 1)


@pytest.mark.parametrize("kind,tier,D", ALL)
def test_pack_unpack_roundtrip(kind, tier, D):
    rng = np.random.default_rng(tier * 10 + D)
    b = TIER_BITS[tier]
    hi = 1 << b
    for n_valid in (T, 5, 1):
        pay = rng.integers(0, hi, (n_valid, D))
        meta = rng.integers(0, 1 << (16 if tier in (4, 5) else 32), (n_valid, D // 32), dtype=np.uint64)
        data = pack_chunk(kind, tier, D, n_valid, pay, meta if tier else None)
        assert data.size == chunk_bytes(tier, D)
        p2, m2 = unpack_chunk(kind, tier, D, data)
        assert np.array_equal(p2[:n_valid], pay)
        assert np.all(p2[n_valid:] == 0)
        if tier:
            assert np.array_equal(m2[:n_valid].astype(np.uint64), meta)
            assert np.all(m2[n_valid:] == 0)


def test_chunk_sizes_d128():
    # K+V bytes per (page, kv head): 16-bit 8192, int8 4608, int4 2560, int2 1536, 1-bit 768, fp8 4352
    assert [2 * chunk_bytes(t, 128) for t in range(6)] == [8192, 4608, 2560, 1536, 768, 4352]
    for t in range(6):
        for D in (64, 128):
            assert chunk_bytes(t, D) % 16 == 0
