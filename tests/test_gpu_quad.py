"""quad page score on the GPU (kvq_quad_build / kvq_quad_append / kvq_quad_page_scores)
vs the oracle's ``oracle.quad``.

The per-page state (lambda bits and the open page's fp64 sums) is compared bit for bit
after the bulk build and after an append; the fp32 scores within the fp32 bound of the
fp64 oracle; then the selected pages and the attention outputs of a whole step scored
by quad.
"""
import numpy as np
import pytest
import torch

from oracle.fp import bits16_to_f64
from oracle.quad import QuadState
from oracle.select import kth_margin
from oracle.step import prepare
from sparse_mixed_precision_kvq_b200 import workloads as W
from tests.parity_helpers import check_output, oracle_step, out_to_f64, query_and_new, sample_units

pytestmark = pytest.mark.gpu

ALL_TIERS = {W.TIER_F16: 0.16, W.TIER_I8: 0.17, W.TIER_I4: 0.17, W.TIER_I2: 0.17, W.TIER_I1: 0.17, W.TIER_F8: 0.16}
CASES = {  # name: (workload, rank, basis kind)
    "c1_r16_random": (lambda: W.small("c1", lens=np.array([2048, 1001])), 16, "random"),
    "c1_r8_law": (lambda: W.small("c1", lens=np.array([700, 2000])), 8, "law"),
    "c0_f16_r32_random": (lambda: W.make("c0", lens=np.array([1000]), append=True, tier_fracs=ALL_TIERS), 32,
                          "random"),
    "c4_r24_random": (lambda: W.small("c4"), 24, "random"),
}
# selection sets must agree where the k-th margin of the oracle's scores exceeds this
# (the fp32 quad term carries a larger rounding error than the plain score)
QUAD_MARGIN = 1e-4


@pytest.fixture(scope="module")
def kvq():
    from sparse_mixed_precision_kvq_b200 import kvq as k
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return k


def _basis(w, rank, kind):
    return np.stack([w.quad_basis(g, rank, kind) for g in range(w.Hkv)])


def _oracle_state(w, basis, b, g, sh):
    return QuadState(sh.korig, sh.L, basis[g].astype(np.float64), w.max_pages)


@pytest.mark.parametrize("name", sorted(CASES))
def test_quad_state_after_build_and_append(kvq, name):
    mk, rank, kind = CASES[name]
    w = mk()
    basis = _basis(w, rank, kind)
    cache = kvq.cache_from_workload(w, quad_basis=basis)
    lam0 = cache.quad.lam.cpu().numpy().view(np.uint16)
    open0 = cache.quad.open.cpu().numpy()
    step = kvq.DecodeStep(w, cache, quad=True)
    step.append()
    torch.cuda.synchronize()
    assert cache.err_bits() == 0, hex(cache.err_bits())
    lam1 = cache.quad.lam.cpu().numpy().view(np.uint16)
    open1 = cache.quad.open.cpu().numpy()
    _, kn, _ = query_and_new(w)
    for b in range(w.B):
        for g in range(w.Hkv):
            sh = prepare(w, b, g)
            qs = _oracle_state(w, basis, b, g, sh)
            P = sh.P
            assert np.array_equal(lam0[b, g, :P], qs.lam_bits[:P]), (b, g)
            if sh.L % 16:
                assert np.array_equal(open0[b, g, 0], qs.s1) and np.array_equal(open0[b, g, 1], qs.s2)
            else:
                assert not open0[b, g].any()
            if w.append:
                pos = int(w.lens[b])
                qs.append(pos, bits16_to_f64(kn[b, g], w.dtype))
                p = pos // 16
                assert np.array_equal(lam1[b, g, :p + 1], qs.lam_bits[:p + 1]), (b, g)
                assert np.array_equal(open1[b, g, 0], qs.s1) and np.array_equal(open1[b, g, 1], qs.s2)


def _score_bound(q_group, summary, lam, basis, s, P):
    """2e-6 of the linear term's magnitude + 3e-5 of the quadratic term's (fp32 dot
    products of D terms, squared)."""
    lin = np.abs(summary[:P]) @ np.abs(q_group).T                        # [P, G]
    zmag = (np.abs(q_group) @ np.abs(basis).T) ** 2                      # [G, r]
    quad = lam[:P] @ zmag.T                                              # [P, G]
    return (2e-6 * s * lin + 3e-5 * 0.5 * s * s * quad).max(axis=1) + 1e-30


@pytest.mark.parametrize("name", sorted(CASES))
def test_quad_step_matches_oracle(kvq, name):
    mk, rank, kind = CASES[name]
    w = mk()
    basis = _basis(w, rank, kind)
    cache = kvq.cache_from_workload(w, quad_basis=basis)
    step = kvq.DecodeStep(w, cache, quad=True)
    step.run()
    torch.cuda.synchronize()
    assert cache.err_bits() == 0, hex(cache.err_bits())
    scores = step.scores.cpu().numpy()
    sel, cnt = step.sel.cpu().numpy(), step.cnt.cpu().numpy()
    out = out_to_f64(step.out, w.dtype)
    q, kn, vn = query_and_new(w)
    compared = 0
    for b in range(w.B):
        for g in range(w.Hkv):
            sh = prepare(w, b, g)
            qs = _oracle_state(w, basis, b, g, sh)
            r = oracle_step(w, sh, b, g, q, kn, vn, quad=qs)
            P = r["P"]
            qg = q[b, g * w.G:(g + 1) * w.G]
            err = np.abs(scores[b, g, :P].astype(np.float64) - r["scores"][:P])
            bound = _score_bound(qg, sh.summary, qs.lam, qs.basis, w.sm_scale, P)
            assert np.all(err <= bound), f"b={b} g={g}: score error {err.max()} (bound {bound[np.argmax(err)]})"
            assert np.all(np.isneginf(scores[b, g, P:]))
            got = sel[b, g, :cnt[b, g]]
            if not np.array_equal(got, r["sel"]):
                m = kth_margin(r["scores"], P, w.k_abs, w.k_frac_bp, w.n_sink, w.n_recent)
                assert m <= QUAD_MARGIN, f"b={b} g={g}: selection differs with margin {m}"
                continue
            compared += 1
            for i in range(w.G):
                check_output(out[b, g * w.G + i], r["out"][i], f"b={b} g={g} h={i}", w.dtype)
    assert compared >= max(1, (w.B * w.Hkv) // 2)


@pytest.mark.parametrize("name", ["c1_r16_random", "c4_r24_random"])
def test_quad_coverage_step_matches_oracle(kvq, name):
    """Coverage selection on quad scores: the mass of page p is n_p * exp(quad_p) (the
    score already carries the softmax scale, so the binding passes sm_scale = 1).  The
    chosen set is the oracle's coverage set on its own quad scores wherever the cut is
    clear of the scores' fp32 rounding (margin 1e-3), and the outputs are the oracle's
    attention over the chosen pages."""
    from oracle.select import coverage_margin, select_coverage
    mk, rank, kind = CASES[name]
    w = mk()
    basis = _basis(w, rank, kind)
    cache = kvq.cache_from_workload(w, quad_basis=basis)
    step = kvq.DecodeStep(w, cache, coverage=0.9, quad=True)
    assert step.params.sm_scale == 1.0
    step.run()
    torch.cuda.synchronize()
    assert cache.err_bits() == 0, hex(cache.err_bits())
    sel, cnt = step.sel.cpu().numpy(), step.cnt.cpu().numpy()
    out = out_to_f64(step.out, w.dtype)
    q, kn, vn = query_and_new(w)
    compared = 0
    for b in range(w.B):
        for g in range(w.Hkv):
            sh = prepare(w, b, g)
            r = oracle_step(w, sh, b, g, q, kn, vn, quad=_oracle_state(w, basis, b, g, sh))
            L, P = int(w.final_lens()[b]), r["P"]
            got = sel[b, g, :cnt[b, g]]
            if coverage_margin(r["scores"], P, L, 1.0, 0.9, w.n_sink, w.n_recent) > 1e-3:
                want = select_coverage(r["scores"], P, L, 1.0, 0.9, w.n_sink, w.n_recent)
                assert list(got) == list(want), (b, g, len(got), len(want))
                compared += 1
            r2 = oracle_step(w, prepare(w, b, g), b, g, q, kn, vn, sel=got.astype(np.int64))
            for i in range(w.G):
                check_output(out[b, g * w.G + i], r2["out"][i], f"quad coverage b={b} g={g} h={i}", w.dtype)
    assert compared >= max(1, (w.B * w.Hkv) // 2)


@pytest.mark.parametrize("name, n_units", [("c1", 8), ("c4", 12)])
def test_quad_full_size_matches_oracle(kvq, name, n_units):
    """The quad-scored step at the workloads' stated sizes (rank 16, the key law's basis;
    c4: ragged rows, whose quad sweep divides only the tiles that hold pages), on a seeded
    sample of units: scores within the bound, -inf past each length, the selected set, and
    every head's output where the set is the oracle's."""
    w = W.make(name)
    basis = _basis(w, 16, "law")
    cache = kvq.cache_from_workload(w, quad_basis=basis)
    step = kvq.DecodeStep(w, cache, quad=True)
    step.run()
    torch.cuda.synchronize()
    assert cache.err_bits() == 0, hex(cache.err_bits())
    scores = step.scores.cpu().numpy()
    sel, cnt = step.sel.cpu().numpy(), step.cnt.cpu().numpy()
    out = out_to_f64(step.out, w.dtype)
    q, kn, vn = query_and_new(w)
    compared = 0
    units = sample_units(w, n_units, seed=3)
    for b, g in units:
        sh = prepare(w, b, g)
        qs = _oracle_state(w, basis, b, g, sh)
        r = oracle_step(w, sh, b, g, q, kn, vn, quad=qs)
        P = r["P"]
        qg = q[b, g * w.G:(g + 1) * w.G]
        err = np.abs(scores[b, g, :P].astype(np.float64) - r["scores"][:P])
        bound = _score_bound(qg, sh.summary, qs.lam, qs.basis, w.sm_scale, P)
        assert np.all(err <= bound), f"b={b} g={g}: score error {err.max()} (bound {bound[np.argmax(err)]})"
        assert np.all(np.isneginf(scores[b, g, P:]))
        got = sel[b, g, :cnt[b, g]]
        if not np.array_equal(got, r["sel"]):
            m = kth_margin(r["scores"], P, w.k_abs, w.k_frac_bp, w.n_sink, w.n_recent)
            assert m <= QUAD_MARGIN, f"b={b} g={g}: selection differs with margin {m}"
            continue
        compared += 1
        for i in range(w.G):
            check_output(out[b, g * w.G + i], r["out"][i], f"{name} b={b} g={g} h={i}", w.dtype)
    assert compared >= max(1, len(units) // 2)


def test_quad_scores_differ_from_the_plain_score(kvq):
    """With a nonzero basis the quadratic term moves the scores off s * (q . kbar)."""
    w = W.small("c1", lens=np.array([1000, 1500]))
    basis = _basis(w, 16, "law")
    cache = kvq.cache_from_workload(w, quad_basis=basis)
    plain = kvq.DecodeStep(w, cache)
    plain.scores_()
    quad = kvq.DecodeStep(w, cache, quad=True)
    quad.scores_()
    torch.cuda.synchronize()
    a = plain.scores.cpu().numpy() * w.sm_scale
    bq = quad.scores.cpu().numpy()
    fin = np.isfinite(a)
    assert np.array_equal(fin, np.isfinite(bq))
    assert np.all(bq[fin] >= a[fin] - 1e-4 * np.abs(a[fin]) - 1e-6)   # the added term is >= 0
    assert np.mean(bq[fin] > a[fin] + 1e-6) > 0.9


@pytest.mark.parametrize("name", ["c1_r16_random", "c4_r24_random"])
def test_fused_quad_append_scores_equals_the_separate_calls(kvq, name):
    """kvq_quad_append_scores (one launch) -> select -> attention gives the bytes, state,
    scores and outputs of kvq_append -> kvq_quad_append -> kvq_quad_page_scores -> ..."""
    mk, rank, kind = CASES[name]
    w = mk()
    basis = _basis(w, rank, kind)
    res = []
    for path in ("calls", "three"):
        cache = kvq.cache_from_workload(w, quad_basis=basis)
        step = kvq.DecodeStep(w, cache, quad=True)
        step.run() if path == "calls" else step.run_three()
        torch.cuda.synchronize()
        assert cache.err_bits() == 0, hex(cache.err_bits())
        res.append(dict(scores=step.scores.cpu().numpy(), sel=step.sel.cpu().numpy(), cnt=step.cnt.cpu().numpy(),
                        out=step.out.cpu().view(torch.int16).numpy(), lam=cache.quad.lam.cpu().numpy().view(np.uint16),
                        open=cache.quad.open.cpu().numpy(), summary=cache.summary.cpu().numpy().view(np.uint16),
                        pools=[None if p is None else p.cpu().numpy() for p in cache.pools]))
    a, b = res
    for key in ("scores", "sel", "cnt", "out", "lam", "open", "summary"):
        assert np.array_equal(a[key], b[key]), key
    for pa, pb in zip(a["pools"], b["pools"]):
        assert (pa is None) == (pb is None) and (pa is None or np.array_equal(pa, pb))
