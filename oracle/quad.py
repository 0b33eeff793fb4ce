"""quad page score: a Gaussian moment-generating-function score from a per-page summary.

Test infrastructure only (see ``oracle/__init__.py``).

AMASS ("What is in the box", Stage A) describes the quad selector as a quadratic,
Gaussian-MGF page score built from a tiny per-page summary that keeps only r'
eigenvalues per page.  The page gives no formula, no r' and no basis.  Reading:

* Model the keys of page p as Gaussian, k ~ N(mu_p, Sigma_p).  The expected
  exponentiated logit of a query q at softmax scale s is then
  ``log E[exp(s q.k)] = s q.mu_p + 1/2 s^2 q^T Sigma_p q`` (the Gaussian MGF).
* ``Sigma_p`` is summarised in a basis U shared by all pages of a kv head: r'
  orthonormal rows u_i (given by the caller, as fp32 values), and page p keeps
  ``lambda_{p,i} = u_i^T Sigma_p u_i`` -- the eigenvalues of Sigma_p when U holds its
  eigenvectors -- so ``q^T Sigma_p q ~= sum_i lambda_{p,i} (u_i . q)^2``.
* ``mu_p`` is the page's fp16 mean-key summary (the same summary the plain score uses);
  ``Sigma_p`` is the page's (1/n) covariance of the keys as they arrived.
* Score of kv head g: the maximum over its query heads, as for the plain score; pages
  at or past the length score -inf.

Arithmetic of the per-page state, fixed so that a page built at once and a page grown
token by token hold the same bits: ``y_{t,i} = sum_d u_{i,d} k_{t,d}`` summed in channel
order, ``S1_i = sum_t y_{t,i}`` and ``S2_i = sum_t y_{t,i}^2`` in token order,
``lambda_{p,i} = fp16(max(S2_i/n - (S1_i/n)^2, 0))``; every step an IEEE fp64 operation
(no fused multiply-add).  The score itself is fp64 here.
"""
from __future__ import annotations

import numpy as np

from .fp import fp16_rne_sat


def projections(keys: np.ndarray, basis: np.ndarray) -> np.ndarray:
    """``y[t, i] = sum_d basis[i, d] * keys[t, d]`` in channel order (fp64)."""
    keys = np.asarray(keys, dtype=np.float64)
    basis = np.asarray(basis, dtype=np.float64)
    y = np.zeros((keys.shape[0], basis.shape[0]))
    for d in range(keys.shape[1]):
        y = y + keys[:, d:d + 1] * basis[None, :, d]
    return y


def moments(y: np.ndarray):
    """Running sums over tokens in order: ``(S1 [r'], S2 [r'])``."""
    s1 = np.zeros(y.shape[1])
    s2 = np.zeros(y.shape[1])
    for t in range(y.shape[0]):
        s1 = s1 + y[t]
        s2 = s2 + y[t] * y[t]
    return s1, s2


def lambdas_from_moments(s1: np.ndarray, s2: np.ndarray, n: int):
    """``fp16(max(S2/n - (S1/n)^2, 0))`` -> (values fp64, fp16 bits, overflow)."""
    m = s1 / n
    v = s2 / n - m * m
    v = np.where(v > 0.0, v, 0.0)
    return fp16_rne_sat(v)


def page_lambdas(keys: np.ndarray, basis: np.ndarray):
    """State of one page from its keys ``[n, D]`` (n >= 1): (lambda values, bits, overflow)."""
    s1, s2 = moments(projections(keys, basis))
    return lambdas_from_moments(s1, s2, keys.shape[0])


class QuadState:
    """quad state of one (sequence, kv head): lambdas of every page and the open page's sums."""

    def __init__(self, korig: np.ndarray, L: int, basis: np.ndarray, P_cap: int):
        T = 16
        r = basis.shape[0]
        self.basis = np.asarray(basis, dtype=np.float64)
        self.lam = np.zeros((P_cap, r))
        self.lam_bits = np.zeros((P_cap, r), np.uint16)
        self.s1 = np.zeros(r)
        self.s2 = np.zeros(r)
        self.overflow = False
        self.L = L
        for p in range((L + T - 1) // T):
            keys = korig[p * T:min(L, p * T + T)]
            s1, s2 = moments(projections(keys, self.basis))
            val, bits, ov = lambdas_from_moments(s1, s2, keys.shape[0])
            self.lam[p], self.lam_bits[p] = val, bits
            self.overflow |= bool(np.any(ov))
            if L % T and p == (L - 1) // T:
                self.s1, self.s2 = s1, s2

    def append(self, pos: int, k: np.ndarray):
        """Token ``pos`` (== current length) with key ``k [D]`` (fp64) joins its page."""
        T = 16
        assert pos == self.L
        p, t = divmod(pos, T)
        y = projections(np.asarray(k, dtype=np.float64)[None], self.basis)[0]
        self.s1 = y.copy() if t == 0 else self.s1 + y
        self.s2 = y * y if t == 0 else self.s2 + y * y
        val, bits, ov = lambdas_from_moments(self.s1, self.s2, t + 1)
        self.lam[p], self.lam_bits[p] = val, bits
        self.overflow |= bool(np.any(ov))
        self.L = pos + 1


def quad_scores(q_group: np.ndarray, summary: np.ndarray, lam: np.ndarray, basis: np.ndarray, sm_scale: float,
                P: int, P_cap: int | None = None) -> np.ndarray:
    """``q_group [G, D]``, ``summary [>=P, D]`` (fp16 values), ``lam [>=P, r']`` (fp16
    values), ``basis [r', D]`` -> scores fp64 ``[P_cap]``:
    ``max_h  s q_h.kbar_p + 1/2 s^2 sum_i lam[p, i] (u_i . q_h)^2``."""
    P_cap = P_cap if P_cap is not None else P
    out = np.full(P_cap, -np.inf)
    if P > 0:
        q = np.asarray(q_group, dtype=np.float64)
        z = (q @ np.asarray(basis, dtype=np.float64).T) ** 2               # [G, r']
        lin = summary[:P] @ q.T                                            # [P, G]
        quad = lam[:P] @ z.T                                               # [P, G]
        out[:P] = (sm_scale * lin + 0.5 * sm_scale * sm_scale * quad).max(axis=1)
    return out
