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
    """Relative gap between the k-th and (k+1)-th best candidate scores (inf if none)."""
    F = forced_pages(P, n_sink, n_recent)
    c = np.array([scores[p] for p in range(P) if p not in F], dtype=np.float64)
    k = min(budget(P, k_abs, k_frac_bp), c.size)
    if k == 0 or k >= c.size:
        return math.inf
    s = np.sort(c)[::-1]
    a, b = s[k - 1], s[k]
    return float((a - b) / max(abs(a), abs(b), 1e-30))
