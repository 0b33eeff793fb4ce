"""Pins of the oracle's quad page score (Gaussian-MGF score from per-page eigenvalues).

* the Gaussian moment-generating function: on many Gaussian keys with a known mean and
  covariance, log-mean-exp of the scaled logits approaches the quad score;
* with U the eigenvectors of a page's covariance, sum_i lambda_i (u_i . q)^2 is
  q^T Sigma q (numpy's covariance), and each lambda is an eigenvalue (numpy's eigh);
* lambda against a two-pass variance written separately; r' = 0 reduces to the scaled
  plain score; a page grown token by token holds the bits of a page built at once.
"""
import numpy as np
import pytest

from oracle.fp import fp16_rne_sat
from oracle.quad import QuadState, page_lambdas, projections, quad_scores
from oracle.score import page_scores


def _orthonormal(rng, r, D):
    q, _ = np.linalg.qr(rng.normal(size=(D, D)))
    return q[:, :r].T.astype(np.float32).astype(np.float64)


def test_gaussian_mgf_closed_form():
    """log E[exp(s q.k)] = s q.mu + 1/2 s^2 q^T Sigma q for k ~ N(mu, Sigma): Monte Carlo
    over 400k keys, lambda from the keys in the eigenbasis of Sigma."""
    rng = np.random.default_rng(0)
    D, n, s = 16, 400_000, 0.25
    ev = np.linspace(0.2, 3.0, D)
    V, _ = np.linalg.qr(rng.normal(size=(D, D)))
    Sigma = (V * ev) @ V.T
    mu = rng.normal(0, 0.5, D)
    keys = rng.multivariate_normal(mu, Sigma, size=n)
    q = rng.normal(size=(1, D))
    lam, _, _ = page_lambdas(keys, V.T)
    got = quad_scores(q, keys.mean(0)[None], lam[None], V.T, s, 1)[0]
    logits = s * (keys @ q[0])
    mc = np.log(np.mean(np.exp(logits - logits.max()))) + logits.max()
    exact = s * q[0] @ mu + 0.5 * s * s * q[0] @ Sigma @ q[0]
    assert abs(mc - exact) < 0.02 * abs(exact) + 0.01        # the MGF itself
    assert abs(got - exact) < 0.02 * abs(exact) + 0.01       # the score estimates it
    assert abs(got - mc) < 0.03 * abs(exact) + 0.01


def test_full_eigenbasis_gives_the_covariance_form():
    rng = np.random.default_rng(1)
    for D, n in ((8, 16), (32, 16), (64, 7)):
        keys = rng.normal(size=(n, D)) * rng.uniform(0.1, 4.0, D) + rng.normal(size=D)
        Sigma = np.cov(keys, rowvar=False, bias=True)
        w, U = np.linalg.eigh(Sigma)
        y = projections(keys, U.T)
        lam = y.var(axis=0)                               # numpy two-pass (1/n) variance
        assert np.allclose(lam, w, rtol=1e-9, atol=1e-9 * w.max())
        q = rng.normal(size=D)
        z = (U.T @ q) ** 2
        assert np.isclose(lam @ z, q @ Sigma @ q, rtol=1e-9)
        val, bits, ov = page_lambdas(keys, U.T)
        want, wbits, _ = fp16_rne_sat(np.maximum(lam, 0.0))
        # the running-sum variance equals the two-pass one to within an fp16 rounding step
        assert np.all(np.abs(val - want) <= np.abs(want) * 2.0 ** -10 + 2.0 ** -24)
        assert not ov.any()


def test_rank_zero_is_the_scaled_plain_score():
    rng = np.random.default_rng(2)
    P, D, G = 9, 32, 4
    summ = rng.normal(size=(P, D)).astype(np.float16).astype(np.float64)
    q = rng.normal(size=(G, D))
    got = quad_scores(q, summ, np.zeros((P, 0)), np.zeros((0, D)), 0.3, P - 2, P)
    want = page_scores(q, summ, P - 2, P)
    assert np.array_equal(got[:P - 2], 0.3 * want[:P - 2]) and np.all(np.isneginf(got[P - 2:]))


def test_quad_term_is_the_max_over_heads_of_each_heads_value():
    rng = np.random.default_rng(3)
    P, D, G, r = 5, 16, 3, 4
    U = _orthonormal(rng, r, D)
    summ = rng.normal(size=(P, D))
    lam = rng.uniform(0, 2, size=(P, r))
    q = rng.normal(size=(G, D))
    s = 0.7
    got = quad_scores(q, summ, lam, U, s, P)
    for p in range(P):
        vals = [s * q[h] @ summ[p] + 0.5 * s * s * sum(lam[p, i] * (U[i] @ q[h]) ** 2 for i in range(r))
                for h in range(G)]
        assert np.isclose(got[p], max(vals), rtol=1e-12)


def test_constant_and_single_token_pages_have_zero_lambda():
    rng = np.random.default_rng(4)
    U = _orthonormal(rng, 4, 16)
    k = rng.normal(size=16)
    for n in (1, 5, 16):
        val, bits, _ = page_lambdas(np.tile(k, (n, 1)), U)
        assert np.all(bits == 0)


@pytest.mark.parametrize("L", [1, 16, 17, 40, 64])
def test_grown_page_equals_built_page(L):
    rng = np.random.default_rng(5)
    D, r = 32, 6
    U = _orthonormal(rng, r, D)
    keys = rng.normal(size=(L + 20, D)).astype(np.float16).astype(np.float64)
    grown = QuadState(keys, L, U, 8)
    for pos in range(L, L + 20):
        grown.append(pos, keys[pos])
    built = QuadState(keys, L + 20, U, 8)
    assert np.array_equal(grown.lam_bits, built.lam_bits)
    if (L + 20) % 16:
        assert np.array_equal(grown.s1, built.s1) and np.array_equal(grown.s2, built.s2)


def test_projection_is_channel_ordered_dot():
    rng = np.random.default_rng(6)
    keys = rng.normal(size=(3, 8))
    U = rng.normal(size=(2, 8))
    y = projections(keys, U)
    for t in range(3):
        for i in range(2):
            acc = 0.0
            for d in range(8):
                acc = acc + U[i, d] * keys[t, d]
            assert y[t, i] == acc


def test_hand_derived_fixture():
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "quad_examples.json")) as f:
        fx = json.load(f)
    for e in fx["cases"]:
        keys, basis = np.array(e["keys"]), np.array(e["basis"])
        lam, _, _ = page_lambdas(keys, basis)
        assert np.allclose(lam, e["lambda"], rtol=1e-6, atol=1e-7), e["why"]
        got = quad_scores(np.array(e["q"]), keys.mean(0)[None], np.array(e["lambda"])[None], basis, e["s"], 1)[0]
        assert np.isclose(got, e["score"], rtol=1e-12), e["why"]
