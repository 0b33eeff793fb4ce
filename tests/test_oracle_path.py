"""Pins for the oracle's summary, score, selection and attention.

Each is checked against something other than itself: textbook formulas written out
separately (math.fsum dot products, scipy softmax), brute force on tiny inputs,
closed forms and invariants of the method.
"""
import math

import numpy as np
import pytest
from scipy.special import logsumexp, softmax

from oracle import cache as ocache
from oracle.attention import attend, lse_combine, token_index
from oracle.fp import bits16_to_f64
from oracle.score import page_scores
from oracle.select import budget, select
from oracle.step import decode_step, prepare, step_pair
from sparse_mixed_precision_kvq_b200 import workloads as W


# ----------------------------------------------------------------- summary / append
def test_summary_is_mean_key_and_single_token_is_key():
    w = W.make("c0", lens=np.array([37]))
    kb, vb = w.keys_bits(0, 0), w.values_bits(0, 0)
    sh = ocache.build(kb, vb, "f16", np.zeros(3, np.int64))
    k = bits16_to_f64(kb, "f16")
    for p in range(3):
        rows = k[p * 16: min(37, p * 16 + 16)]
        assert np.array_equal(sh.summary[p], np.float16(rows.mean(0)).astype(np.float64))
    assert np.array_equal(sh.summary[2][None], np.float16(k[32:37].mean(0))[None].astype(np.float64))
    one = ocache.build(kb[:1], vb[:1], "f16", np.zeros(1, np.int64))
    assert np.array_equal(one.summary[0], k[0])          # fp16 input: n = 1 gives the key back


@pytest.mark.parametrize("tier", [0, 1, 2, 3, 4])
def test_append_equals_build(tier):
    """Growing a page token by token gives the same summary, sums and bytes as building it."""
    w = W.make("c1", B=1, lens=np.array([45]), append=False)
    kb, vb = w.keys_bits(0, 2), w.values_bits(0, 2)
    tiers = np.full(3, tier)
    full = ocache.build(kb, vb, "bf16", tiers)
    grown = ocache.build(kb[:16], vb[:16], "bf16", tiers, capacity_pages=3)
    for pos in range(16, 45):
        ocache.append(grown, pos, kb[pos], vb[pos])
    assert np.array_equal(full.summary_bits[:3], grown.summary_bits[:3])
    assert np.array_equal(full.ksum, grown.ksum)
    for p in range(3):
        for kind in "kv":
            assert np.array_equal(ocache.page_bytes(full, p, kind), ocache.page_bytes(grown, p, kind))


# ----------------------------------------------------------------- score
def test_score_is_max_over_group_of_textbook_dots():
    rng = np.random.default_rng(0)
    G, D, P = 4, 64, 9
    q = rng.standard_normal((G, D))
    summ = rng.standard_normal((P + 3, D))
    s = page_scores(q, summ, P, P + 3)
    for p in range(P):
        want = max(math.fsum(q[h, j] * summ[p, j] for j in range(D)) for h in range(G))
        assert abs(s[p] - want) <= 1e-12 * max(1.0, abs(want))
    assert np.all(np.isneginf(s[P:]))
    eq = page_scores(q, np.tile(summ[:1], (P, 1)), P)
    assert np.all(eq == eq[0])


# ----------------------------------------------------------------- select
def _brute_select(scores, P, k, n_sink, n_recent):
    forced = {p for p in range(P) if p < n_sink or p >= P - n_recent}
    cand = [p for p in range(P) if p not in forced]
    k = min(k, len(cand))

    def beats(a, b):   # does candidate a rank before candidate b?
        sa, sb = scores[a], scores[b]
        na, nb = math.isnan(sa), math.isnan(sb)
        if na != nb:
            return nb
        if not na and sa != sb:
            return sa > sb
        return a < b
    chosen = {p for p in cand if sum(beats(o, p) for o in cand if o != p) < k}
    return sorted(forced | chosen)


def test_select_matches_bruteforce_with_ties_and_nans():
    rng = np.random.default_rng(1)
    for trial in range(300):
        P = int(rng.integers(0, 24))
        s = rng.integers(-3, 4, P).astype(np.float64)     # many ties
        if P and trial % 5 == 0:
            s[rng.integers(0, P)] = np.nan
        k = int(rng.integers(0, 8))
        ns, nr = int(rng.integers(0, 3)), int(rng.integers(0, 4))
        got = select(s, P, k, 0, ns, nr)
        assert list(got) == _brute_select(s, P, k, ns, nr), (P, k, ns, nr, s)
        assert list(got) == sorted(set(got))


def test_select_budget_and_forced():
    s = np.arange(100, dtype=np.float64)[::-1].copy()           # page 0 best
    assert budget(2048, -1, 500) == 103 and budget(2049, -1, 1000) == 205
    assert budget(8193, -1, 500) == 410 and budget(10, 3, 500) == 3
    sel = select(s, 100, -1, 500, 1, 4)                          # 5 % of 100 = 5
    assert list(sel) == [0, 1, 2, 3, 4, 5, 96, 97, 98, 99]
    allp = select(s, 100, 1000, 0, 1, 4)
    assert list(allp) == list(range(100))
    tie = select(np.zeros(10), 10, 3, 0, 0, 0)
    assert list(tie) == [0, 1, 2]                                # equal scores -> lower index


def test_planted_pages_always_selected():
    """c0: the four planted pages are always among the selected pages."""
    w = W.make("c0")
    res = decode_step(w)
    for g in range(w.Hkv):
        planted = set(w.planted_pages(0))
        assert planted <= set(res[(0, g)]["sel"])
        assert len(res[(0, g)]["sel"]) == 10


# ----------------------------------------------------------------- attention
def test_all_pages_16bit_equals_textbook_dense_attention():
    w = W.make("c0", lens=np.array([300]))
    sh = prepare(w, 0, 1)
    q = bits16_to_f64(w.query_bits(), w.dtype)[0]
    P = sh.P
    idx = token_index(np.arange(P), sh.L)
    k = bits16_to_f64(w.keys_bits(0, 1), "f16")
    v = bits16_to_f64(w.values_bits(0, 1), "f16")
    for h in range(4, 8):
        o, lse, _, _ = attend(q[h], sh.khat[idx], sh.vhat[idx], w.sm_scale)
        logits = (k @ q[h]) / math.sqrt(w.D)
        want = softmax(logits) @ v
        assert np.allclose(o, want, rtol=1e-12, atol=1e-13)
        assert abs(lse - logsumexp(logits)) < 1e-12


def test_single_token_and_identical_keys():
    rng = np.random.default_rng(4)
    q = rng.standard_normal(16)
    k = rng.standard_normal((1, 16))
    v = rng.standard_normal((1, 16))
    o, lse, _, _ = attend(q, k, v, 0.25)
    assert np.array_equal(o, v[0]) and abs(lse - 0.25 * float(k[0] @ q)) < 1e-12
    kk = np.tile(k, (7, 1))
    vv = rng.standard_normal((7, 16))
    o, lse, _, _ = attend(q, kk, vv, 0.25)
    assert np.allclose(o, vv.mean(0), rtol=1e-13, atol=1e-14)
    assert abs(lse - (0.25 * float(k[0] @ q) + math.log(7))) < 1e-12


def test_split_combine_equals_unsplit():
    rng = np.random.default_rng(9)
    q = rng.standard_normal(32)
    k = rng.standard_normal((200, 32)) * 3
    v = rng.standard_normal((200, 32))
    o, lse, _, _ = attend(q, k, v, 0.3)
    for cuts in ([0, 200], [0, 1, 200], [0, 50, 51, 120, 200], list(range(0, 201, 10))):
        parts = []
        for a, b in zip(cuts[:-1], cuts[1:]):
            oi, _, mi, li = attend(q, k[a:b], v[a:b], 0.3)
            parts.append((oi, mi, li))
        oc, lc = lse_combine(parts)
        assert np.allclose(oc, o, rtol=1e-13, atol=1e-13) and abs(lc - lse) < 1e-12


def test_quantised_pages_attend_dequantised_values():
    """A quantised page is attended through the values it reads back, not the originals."""
    w = W.make("c4", B=1, lens=np.array([70]), append=False,
               tier_fracs={W.TIER_I2: 1.0})
    sh = prepare(w, 0, 0)
    assert np.all(sh.tiers[:5] == W.TIER_I2)
    k = bits16_to_f64(w.keys_bits(0, 0), "bf16")
    assert not np.array_equal(sh.khat[:70], k)
    err = np.abs(sh.khat[:70] - k)
    assert err.max() > 0 and np.all(np.isfinite(sh.khat[:70]))


def test_step_pair_with_given_selection():
    w = W.small("c2")
    q = bits16_to_f64(w.query_bits(), w.dtype)
    kn, vn = w.new_kv_bits()
    sh = prepare(w, 1, 3)
    r = step_pair(w, sh, 1, 3, q[1], kn[1, 3], vn[1, 3], sel=[0, 5, 62])
    assert list(r["used"]) == [0, 5, 62] and r["L"] == 1001
    assert r["out"].shape == (4, 128) and np.all(np.isfinite(r["out"]))


def test_large_logits_and_empty_selection():
    """Logits of magnitude ~1e3 stay finite and equal scipy's softmax / logsumexp; an empty
    token set gives zeros and lse = -inf, and drops out of the combine."""
    rng = np.random.default_rng(12)
    q = rng.standard_normal(16) * 40
    k = rng.standard_normal((50, 16)) * 40
    v = rng.standard_normal((50, 16))
    o, lse, _, _ = attend(q, k, v, 0.25)
    logits = 0.25 * (k @ q)
    assert np.abs(logits).max() > 500
    assert np.allclose(o, softmax(logits) @ v, rtol=1e-12, atol=1e-13)
    assert abs(lse - logsumexp(logits)) < 1e-9 * abs(lse)
    oe, lse_e, me, le = attend(q, k[:0], v[:0], 0.25)
    assert np.array_equal(oe, np.zeros(16)) and lse_e == -np.inf and le == 0.0
    oc, lc = lse_combine([(oe, me, le), (o, *attend(q, k, v, 0.25)[2:])])
    assert np.allclose(oc, o, rtol=1e-13) and abs(lc - lse) < 1e-9 * abs(lse)
