"""Pins of two small oracle functions that decide what the GPU parity tests accept.

* ``dequant_sign``: the 1-bit tier's read-back.  ARGUS "Visual Architecture" names a
  1-bit tier, 8 signs packed per byte; the reading used throughout is x >= 0 -> +m,
  otherwise -m, with m the group's fp16 mean magnitude.  Checked against hand-written
  bits and magnitudes (``tests/golden/quant_examples.json``) and against signs and
  magnitudes computed here directly from x, without the oracle's quantiser.
* ``kth_margin``: the relative gap between the k-th and (k+1)-th best candidates, which
  excuses a selection mismatch only when it is at most 1e-5.  Checked against margins
  worked out by hand and against what the gap means for the selection itself: scores
  moved by less than the gap never change the selected set, and swapping the two scores
  at the cut always does.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle.quant import GROUP, TIER_I1, dequant_sign, quantise_sign, quantise_token
from oracle.select import kth_margin, select

GOLD = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ 1-bit read-back
def test_sign_readback_golden():
    with open(os.path.join(GOLD, "quant_examples.json")) as f:
        cases = [c for c in json.load(f)["cases"] if c["bits"] == 1]
    assert len(cases) >= 2
    for c in cases:
        bits = np.array(c["codes"], dtype=np.int64)[None]
        m = np.array([c["m"]])
        assert list(dequant_sign(bits, m)[0]) == c["xhat"], c["name"]
        x = np.array(c["x"], dtype=np.float64)
        assert list(quantise_token(x, TIER_I1)["xhat"]) == c["xhat"], c["name"]


def test_sign_readback_hand_bits():
    """Bit 1 reads back +m, bit 0 reads back -m, per group's own magnitude."""
    bits = np.array([[1, 0, 0, 1] * 8, [0] * 32, [1] * 32])
    m = np.array([0.75, 2.0, 0.0])
    got = dequant_sign(bits, m)
    assert list(got[0, :4]) == [0.75, -0.75, -0.75, 0.75]
    assert np.all(got[1] == -2.0)
    assert np.all(got[2] == 0.0)


def test_sign_readback_is_alpha_times_sign_of_x():
    """x_hat = m * sign(x) with sign(+-0) = +, m = fp16(sum|x| / 32), computed here from
    x alone (math.fsum, numpy's fp16 rounding), never from the quantiser's bits."""
    rng = np.random.default_rng(11)
    x = rng.standard_normal((200, GROUP)).astype(np.float16).astype(np.float64)
    x[0, :4] = [-0.0, 0.0, -1.0, 1.0]
    x[1] = -np.abs(x[1])                                   # every sign negative
    want_m = np.array([float(np.float16(math.fsum(abs(v) for v in row) / GROUP)) for row in x])
    want = np.where(x >= 0.0, 1.0, -1.0) * want_m[:, None]
    got = quantise_token(x.reshape(-1), TIER_I1)["xhat"].reshape(x.shape)
    assert np.array_equal(got, want)
    assert got[0, 0] == want_m[0] and got[0, 2] == -want_m[0]
    bits, m, _, _ = quantise_sign(x)
    assert np.array_equal(dequant_sign(bits, m), want)


# ------------------------------------------------------------------ k-th margin
@pytest.mark.parametrize("scores, P, k_abs, k_bp, ns, nr, want", [
    ([10, 5, 4, 3, 1, 0], 6, 2, 0, 0, 0, 0.2),            # clear gap: (5 - 4) / 5
    ([3, 7, 7, 1], 4, 1, 0, 0, 0, 0.0),                    # exact tie at the cut
    ([3, 7, 7, 1], 4, 2, 0, 0, 0, (7 - 3) / 7),
    ([3, 7, 7, 1], 4, 0, 0, 0, 0, math.inf),               # k = 0: no cut
    ([3, 7, 7, 1], 4, 4, 0, 0, 0, math.inf),               # k >= |C|: every candidate chosen
    ([3, 7, 7, 1], 4, 9, 0, 0, 0, math.inf),
    ([100, 2, 9, 5, 4, -50], 6, 2, 0, 1, 1, 0.2),          # forced pages 0 and 5 are not candidates
    ([100, 2, 9, 5, 4, -50], 6, 3, 0, 1, 1, (4 - 2) / 4),
    (list(range(10)), 10, -1, 2500, 0, 0, 1 / 7),          # k = ceil(10 * 0.25) = 3: (7 - 6) / 7
    (list(range(10)), 10, -1, 2000, 0, 0, 1 / 8),          # k = 2: (8 - 7) / 8
    ([-1, -2, -4], 3, 1, 0, 0, 0, 0.5),                    # negative scores: (-1 + 2) / 2
    ([0.0, 0.0, -1e-40], 3, 2, 0, 0, 0, 1e-10),            # denominator floor: 1e-40 / 1e-30
    ([math.nan, 5, 3, 1], 4, 1, 0, 0, 0, 0.4),             # NaN ranks lowest: (5 - 3) / 5
    ([math.nan, 5, 3, 1], 4, 3, 0, 0, 0, math.inf),        # cut between 1 and NaN
    ([math.nan, 5, math.nan], 3, 2, 0, 0, 0, math.inf),    # NaNs ordered by page only
    ([math.inf, 5, 3], 3, 1, 0, 0, 0, math.inf),           # inf vs a number
    ([math.inf, math.inf, 3], 3, 1, 0, 0, 0, 0.0),         # inf tie
    ([2, -math.inf, -math.inf], 3, 2, 0, 0, 0, 0.0),
])
def test_kth_margin_hand_values(scores, P, k_abs, k_bp, ns, nr, want):
    s = np.array(scores, dtype=np.float64)
    got = kth_margin(s, P, k_abs, k_bp, ns, nr)
    if math.isinf(want):
        assert math.isinf(got) and got > 0
    else:
        assert got == pytest.approx(want, rel=1e-12, abs=0.0)


def test_kth_margin_bounds_the_selection():
    """A relative move of every candidate's score by less than half the margin keeps the
    selected set; exchanging the k-th and (k+1)-th scores changes it unless they are equal."""
    rng = np.random.default_rng(7)
    checked = swapped = 0
    for trial in range(400):
        P = int(rng.integers(2, 40))
        s = rng.standard_normal(P) * 10 ** rng.uniform(-3, 3)
        if trial % 7 == 0:
            s[rng.integers(0, P)] = s[rng.integers(0, P)]          # a duplicate
        k, ns, nr = int(rng.integers(0, P)), int(rng.integers(0, 3)), int(rng.integers(0, 3))
        base = select(s, P, k, 0, ns, nr)
        m = kth_margin(s, P, k, 0, ns, nr)
        assert m >= 0
        if m > 0:
            eps = min(m, 1.0) * 0.49
            for _ in range(5):
                t = s * (1 + eps * rng.uniform(-1, 1, P) / 2)
                assert list(select(t, P, k, 0, ns, nr)) == list(base), (trial, m)
            checked += 1
        forced = set(range(min(ns, P))) | set(range(max(0, P - nr), P))
        cand = [p for p in range(P) if p not in forced]
        kk = min(k, len(cand))
        if 0 < kk < len(cand):
            order = sorted(cand, key=lambda p: (-s[p], p))
            pa, pb = order[kk - 1], order[kk]
            t = s.copy()
            t[pa], t[pb] = s[pb], s[pa]
            if s[pa] != s[pb]:
                assert list(select(t, P, k, 0, ns, nr)) != list(base)
                swapped += 1
            else:
                assert m == 0.0
    assert checked > 100 and swapped > 100
