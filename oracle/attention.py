"""Attention of one query head over the tokens of the selected pages.

Test infrastructure only (see ``oracle/__init__.py``).

AMASS ("What is in the box"): a sparse paged kernel reads only the selected pages.
ARGUS ("Why It Works: Storage vs. Computation"): stored low-bit values are turned
back into high-precision values before attention; no low-bit arithmetic enters the
attention itself.  So for query head h of kv head g = h // G, over the tokens
``t in U_{p in S} [p*T, min(p*T + T, len))`` (pages ascending, tokens ascending):

    l_t = sm_scale * q_h . khat_t,   m = max_t l_t,   w_t = exp(l_t - m)
    o   = sum_t w_t vhat_t / sum_t w_t,               lse = m + ln(sum_t w_t)

``khat``/``vhat`` are the values read back from storage.  The softmax scale
defaults to 1/sqrt(D).  In fp64.  A partition of the tokens can be attended part by
part and merged with the log-sum-exp combine ``lse_combine``.
"""
from __future__ import annotations

import numpy as np

from .layout import T


def token_index(sel: np.ndarray, L: int) -> np.ndarray:
    idx = [np.arange(p * T, min(p * T + T, L)) for p in np.asarray(sel, dtype=np.int64)]
    return np.concatenate(idx) if idx else np.zeros(0, dtype=np.int64)


def attend(q: np.ndarray, khat: np.ndarray, vhat: np.ndarray, sm_scale: float):
    """``q [D]``, ``khat/vhat [N, D]`` -> ``(o [D], lse, m, l)`` (unnormalised parts too)."""
    if khat.shape[0] == 0:
        return np.zeros(q.shape[-1]), -np.inf, -np.inf, 0.0
    logits = sm_scale * (khat @ q)
    m = logits.max()
    w = np.exp(logits - m)
    l = w.sum()
    o = (w @ vhat) / l
    return o, m + np.log(l), m, l


def lse_combine(parts):
    """Merge partial results ``[(o_i (normalised), m_i, l_i), ...]`` of disjoint token sets."""
    parts = [p for p in parts if p[2] > 0]
    if not parts:
        return None, -np.inf
    M = max(p[1] for p in parts)
    L = sum(p[2] * np.exp(p[1] - M) for p in parts)
    o = sum(p[0] * p[2] * np.exp(p[1] - M) for p in parts) / L
    return o, M + np.log(L)
