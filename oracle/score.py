"""Page score from the mean-key summary.

Test infrastructure only (see ``oracle/__init__.py``).

AMASS ("What is in the box") selects pages by "a compact per-page score" built from
the page summary; its "quad" score is not specified on the page, so the plainest
score is used: the query-summary dot product ``q_h . kbar_p``.  Pages are selected
per kv head, and a kv head serves its G query heads, so the page score of kv head g
is the maximum over those heads:

    s[g, p] = max_{h in [g*G, g*G + G)}  sum_j q[h, j] * kbar[g, p, j]

No softmax scale is applied (a positive factor does not change the order).  Pages at
or past the sequence length score -inf.  Computed in fp64.
"""
from __future__ import annotations

import numpy as np


def page_scores(q_group: np.ndarray, summary: np.ndarray, P: int, P_cap: int | None = None) -> np.ndarray:
    """``q_group [G, D]`` fp64, ``summary [>=P, D]`` fp64 -> scores fp64 ``[P_cap]``."""
    P_cap = P_cap if P_cap is not None else P
    out = np.full(P_cap, -np.inf)
    if P > 0:
        dots = summary[:P] @ np.asarray(q_group, dtype=np.float64).T   # [P, G]
        out[:P] = dots.max(axis=1)
    return out
