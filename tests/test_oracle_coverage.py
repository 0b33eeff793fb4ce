"""Pins of the oracle's coverage (nucleus) selection against brute force and closed forms."""
import itertools
import math

import numpy as np
import pytest

from oracle.select import coverage_margin, forced_pages, page_masses, select_coverage


def _brute(scores, P, L, scale, cov, ns, nr):
    """Smallest number of candidates whose mass, with the forced pages', reaches the target,
    found over every subset; and the largest mass any subset of that size reaches."""
    m = page_masses(scores, P, L, scale)
    F = forced_pages(P, ns, nr)
    C = [p for p in range(P) if p not in F]
    target = cov * math.fsum(m)
    base = math.fsum(m[p] for p in F)
    for k in range(len(C) + 1):
        best = max((math.fsum(m[p] for p in sub) for sub in itertools.combinations(C, k)), default=0.0)
        if base + best >= target:
            return k, base + best
    return len(C), None


@pytest.mark.parametrize("seed", range(40))
def test_coverage_is_smallest_and_heaviest(seed):
    rng = np.random.default_rng(seed)
    P = int(rng.integers(1, 10))
    L = 16 * (P - 1) + int(rng.integers(1, 17))
    scores = rng.normal(0, 3, P).astype(np.float32)
    if seed % 5 == 0:
        scores = np.round(scores).astype(np.float32)  # ties
    cov = float(rng.choice([0.5, 0.8, 0.95, 0.99]))
    ns, nr = int(rng.integers(0, 2)), int(rng.integers(0, 2))
    got = select_coverage(scores, P, L, 1.0, cov, ns, nr)
    F = forced_pages(P, ns, nr)
    k_brute, best = _brute(scores, P, L, 1.0, cov, ns, nr)
    chosen = [p for p in got if p not in F]
    assert len(chosen) == k_brute
    m = page_masses(scores, P, L, 1.0)
    assert F <= set(got.tolist())
    if best is not None:  # the greedy set is as heavy as the best subset of its size
        assert math.isclose(math.fsum(m[p] for p in got), best, rel_tol=1e-12)


def test_equal_scores_closed_form():
    P, L = 40, 16 * 40
    scores = np.full(P, 2.5, np.float32)
    for cov in (0.5, 0.9, 0.95):
        got = select_coverage(scores, P, L, 0.3, cov, 1, 2)
        # every page has mass 16: the forced 3 plus the fewest others reaching cov * 40 pages
        k = max(0, math.ceil(cov * P - 1e-9) - 3)
        assert got.size == 3 + k
        # ties go to the lower page index: the candidates chosen are pages 1 .. k
        assert list(got[1:1 + k]) == list(range(1, 1 + k))


def test_extremes_and_shift_invariance():
    rng = np.random.default_rng(3)
    P, L = 30, 16 * 29 + 5
    s = rng.integers(-6, 7, P).astype(np.float32)
    assert list(select_coverage(s, P, L, 1.0, 0.0, 0, 0)) == []
    assert list(select_coverage(s, P, L, 1.0, 0.0, 1, 1)) == [0, P - 1]
    assert select_coverage(s, P, L, 1.0, 1.0, 0, 0).size == P
    # a very sharp softmax keeps exactly the top-scoring pages (the others have no mass left)
    top = np.flatnonzero(s == s.max())
    assert list(select_coverage(s, P, L, 80.0, 0.95, 0, 0)) == list(top)
    # adding a constant to every score changes no mass
    assert list(select_coverage(s + 7, P, L, 0.5, 0.9, 1, 2)) == list(select_coverage(s, P, L, 0.5, 0.9, 1, 2))


def test_last_page_mass_uses_its_valid_tokens_and_nan_has_none():
    P, L = 4, 16 * 3 + 1          # the last page holds one token
    s = np.array([0.0, 0.0, 0.0, 2.0], np.float32)
    m = page_masses(s, P, L, 1.0)
    assert m[3] == 1.0 and np.allclose(m[:3], 16 * math.exp(-2.0))
    s2 = np.array([np.nan, 1.0, 0.0, 0.0], np.float32)
    assert page_masses(s2, P, L, 1.0)[0] == 0.0
    assert 0 not in select_coverage(s2, P, L, 1.0, 0.99, 0, 0)


def test_margin_is_small_only_near_a_decision():
    P, L = 8, 128
    s = np.array([5, 4, 3, 2, 1, 0, -1, -2], np.float32)
    assert coverage_margin(s, P, L, 1.0, 0.9, 0, 0) > 1e-3
    m = page_masses(s, P, L, 1.0)
    cut = math.fsum(m[:2]) / math.fsum(m)   # covering exactly the top two pages
    assert coverage_margin(s, P, L, 1.0, cut, 0, 0) < 1e-12


def test_zero_mass_pages_are_never_needed():
    """With coverage 1 the target is the total mass, which the positive masses reach in
    exact arithmetic; pages of zero mass (NaN scores) are never chosen, every page of
    positive mass is.  The seed is one where the fp64 running sum of the sorted positive
    masses ends 3.6e-15 short of fsum of all masses, so a loop that only compared the
    running sum with the target would go on into the NaN pages."""
    rng = np.random.default_rng(2)
    P, L = 24, 16 * 24
    s = rng.normal(0, 3, P).astype(np.float32)
    s[rng.integers(0, P, 5)] = np.nan
    m = page_masses(s, P, L, 1.0)
    F = forced_pages(P, 1, 1)
    order = sorted((p for p in range(P) if p not in F), key=lambda p: (-m[p], p))
    covered = math.fsum(m[p] for p in F)
    for p in order:
        if m[p] > 0:
            covered += m[p]
    assert covered < math.fsum(m)  # the rounding this case is chosen for
    got = set(select_coverage(s, P, L, 1.0, 1.0, 1, 1).tolist())
    assert got == F | {p for p in range(P) if m[p] > 0}
    assert not any(np.isnan(s[p]) for p in got - F)
    # the same pages without the NaNs: every page
    s2 = np.where(np.isnan(s), np.float32(-1.0), s)
    assert select_coverage(s2, P, L, 1.0, 1.0, 1, 1).size == P
