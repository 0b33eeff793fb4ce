"""Top-k page selection with forced sink and recent pages.

Test infrastructure only (see ``oracle/__init__.py``).

* AMASS ("Quickstart", ``budget``): a fixed fraction of the pages is selected.  The
  fraction is applied per sequence and rounded up in integer arithmetic:
  ``k = ceil(P * bp / 10000)`` for a fraction of ``bp`` basis points, or an absolute k.
* ARGUS ("Quickstart", ``sink_tokens``; "The One-Minute Explanation": recent tokens
  stay hot): the first ``n_sink`` pages and the last ``n_recent`` pages are always
  attended, in addition to the top k (they do not count against it).
* The remaining candidates are ranked by score (higher first), ties broken by the
  lower page index; a NaN score ranks below every number.

The selected set is returned in ascending page order.
"""
from __future__ import annotations

import math

import numpy as np


def budget(P: int, k_abs: int, k_frac_bp: int) -> int:
    if k_abs >= 0:
        return k_abs
    return (P * k_frac_bp + 9999) // 10000


def forced_pages(P: int, n_sink: int, n_recent: int) -> set:
    f = set(range(0, min(n_sink, P)))
    f |= set(range(max(0, P - n_recent), P))
    return f


def select(scores: np.ndarray, P: int, k_abs: int, k_frac_bp: int, n_sink: int,
           n_recent: int) -> np.ndarray:
    """Selected pages of one (sequence, kv head), ascending, int64."""
    F = forced_pages(P, n_sink, n_recent)
    C = [p for p in range(P) if p not in F]
    k = min(budget(P, k_abs, k_frac_bp), len(C))

    def rank_key(p):
        s = float(scores[p])
        s_key = -math.inf if math.isnan(s) else s
        nan_last = 1 if math.isnan(s) else 0
        return (nan_last, -s_key, p)

    top = sorted(C, key=rank_key)[:k]
    return np.array(sorted(F | set(top)), dtype=np.int64)


def kth_margin(scores: np.ndarray, P: int, k_abs: int, k_frac_bp: int, n_sink: int,
               n_recent: int) -> float:
    """Relative gap between the k-th and (k+1)-th best candidate scores, in the order the
    selection ranks them (NaN below every number): ``(a - b) / max(|a|, |b|, 1e-30)``.

    inf when no cut exists (k = 0 or every candidate chosen) or when the cut cannot move
    under a rounding of the scores: ``b`` is NaN (a NaN never outranks a number and NaNs
    are ordered by page index alone), or exactly one of ``a``, ``b`` is infinite.  Equal
    scores (an exact tie, infinite ones included) give 0."""
    F = forced_pages(P, n_sink, n_recent)
    c = [float(scores[p]) for p in range(P) if p not in F]
    k = min(budget(P, k_abs, k_frac_bp), len(c))
    if k == 0 or k >= len(c):
        return math.inf
    s = sorted(c, key=lambda v: (1, 0.0) if math.isnan(v) else (0, -v))
    a, b = s[k - 1], s[k]
    if math.isnan(b):
        return math.inf
    if a == b:
        return 0.0
    if math.isinf(a) or math.isinf(b):
        return math.inf
    return float((a - b) / max(abs(a), abs(b), 1e-30))


# ----------------------------------------------------------------------------- coverage
# AMASS "Quickstart" (``coverage=0.95``: the nucleus variant of the selection).  The pages
# do not give the mass estimate; the plainest reading, used here: a page's attention mass
# is estimated from its score as ``n_p * exp(sm_scale * s_p)`` (n_p = the page's valid
# tokens, the score standing in for each token's logit), normalised over all pages of the
# (sequence, kv head).  The forced pages are attended and count as covered; candidates are
# then added by estimated mass (larger first, lower page index first on ties) until the
# covered mass reaches ``coverage`` of the total.  A NaN score has mass 0, and pages of
# zero mass are never added (in exact arithmetic the positive masses reach any target up
# to the total).

def page_masses(scores: np.ndarray, P: int, L: int, sm_scale: float) -> np.ndarray:
    """Estimated mass of pages 0..P-1 (fp64), relative to the largest score's page."""
    s = np.asarray(scores[:P], dtype=np.float64)
    n = np.full(P, 16.0)
    if P:
        n[P - 1] = float(L - 16 * (P - 1))
    finite = s[~np.isnan(s)]
    if finite.size == 0:
        return np.zeros(P)
    smax = float(finite.max())
    m = np.zeros(P)
    for p in range(P):
        if not math.isnan(s[p]):
            m[p] = n[p] * math.exp(sm_scale * (s[p] - smax))
    return m


def select_coverage(scores: np.ndarray, P: int, L: int, sm_scale: float, coverage: float, n_sink: int,
                    n_recent: int) -> np.ndarray:
    """Coverage selection of one (sequence, kv head), ascending, int64.

    Candidates of zero mass (NaN or underflowed scores) are never added: they come last in
    the mass order, and with coverage <= 1 the positive masses reach the target in exact
    arithmetic, so the running fp64 sum can stop short of it only by rounding (at coverage
    1), where adding pages that carry no mass would not be the rule's choice."""
    F = forced_pages(P, n_sink, n_recent)
    m = page_masses(scores, P, L, sm_scale)
    total = math.fsum(m)
    covered = math.fsum(m[p] for p in F)
    target = coverage * total
    order = sorted((p for p in range(P) if p not in F), key=lambda p: (-m[p], p))
    chosen = []
    for p in order:
        if covered >= target or m[p] == 0.0:
            break
        chosen.append(p)
        covered += m[p]
    return np.array(sorted(F | set(chosen)), dtype=np.int64)


def coverage_margin(scores: np.ndarray, P: int, L: int, sm_scale: float, coverage: float, n_sink: int,
                    n_recent: int) -> float:
    """How far the coverage cut is from being decided otherwise: the smaller of the relative
    gap between the last chosen and the first unchosen candidate masses and the relative
    distance of the covered mass (before the last chosen page) from the target."""
    F = forced_pages(P, n_sink, n_recent)
    m = page_masses(scores, P, L, sm_scale)
    total = math.fsum(m)
    target = coverage * total
    order = sorted((p for p in range(P) if p not in F), key=lambda p: (-m[p], p))
    covered = math.fsum(m[p] for p in F)
    k = 0
    while k < len(order) and covered < target and m[order[k]] > 0.0:
        covered += m[order[k]]
        k += 1
    out = math.inf
    if 0 < k < len(order):
        a, b = m[order[k - 1]], m[order[k]]
        out = min(out, (a - b) / max(a, 1e-300))
    if total > 0:
        before = covered - (m[order[k - 1]] if k else 0.0)
        out = min(out, abs(target - before) / total, abs(covered - target) / total)
    return float(out)
