"""GPU path vs the CPU oracle at the workloads' stated sizes, and in the attention
kernel's deep-pipeline regime.

* Full size: c1, c2, c3 and c4 with their own batch, heads and context (Llama-3-8B- and
  Qwen2.5-3B-shaped layers at 32k / 131k / ragged 2k-64k context), run through the four
  C-ABI calls (c1 and c4 also through the one-launch fused step, c2 and c4 through
  kvq_append_scores + select + attention).  A seeded sample of (sequence,
  kv head) units -- always the first and the last, and for c4 the longest and the
  shortest sequence -- is checked against the oracle's step: every page's bytes after the
  append, summaries, open-page key sums, scores, the selected set (bit-exact where the
  k-th margin exceeds 1e-5) and every query head's output and lse.  At these sizes each
  warp of the attention kernel streams 2-12 pages, so its copy ring wraps, its mbarriers
  are reused with flipped phase, and segments end and begin inside a warp.
* Deep pipeline on small batches: the attention grid is cut to 1-7 CTAs
  (kvq_set_grid_override), so each warp takes 2-24 pages and segments split across CTAs
  in every way; and one batch selects every page (k = 100 %) at the default grid, 7-14
  pages per warp, in 16-bit and in all six tiers.
* Failure detection: a bounded wait that runs out.  With a 1 ms limit in the workspace
  and the fused step's work queue started past its score items (host-side setup only),
  the attention items wait for selections that never come; the call returns with
  KVQ_DERR_TIMEOUT set, and the re-initialised workspace then gives a correct step.
"""
import time

import numpy as np
import pytest
import torch

from oracle.step import prepare
from sparse_mixed_precision_kvq_b200 import workloads as W
from tests.parity_helpers import (check_pages, check_summary, check_unit, out_to_f64, query_and_new, sample_units,
                                  snapshot)

pytestmark = pytest.mark.gpu

ALL_TIERS = {W.TIER_F16: 0.16, W.TIER_I8: 0.17, W.TIER_I4: 0.17, W.TIER_I2: 0.17, W.TIER_I1: 0.17, W.TIER_F8: 0.16}


@pytest.fixture(scope="module")
def kvq():
    from sparse_mixed_precision_kvq_b200 import kvq as k
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return k


def _results(step, w):
    torch.cuda.synchronize()
    return dict(scores=step.scores.cpu().numpy(), sel=step.sel.cpu().numpy(), cnt=step.cnt.cpu().numpy(),
                out=out_to_f64(step.out, w.dtype), lse=step.lse.cpu().numpy())


def _check_units(w, cache, res, units, what, tail=True):
    snap = snapshot(cache)
    q, kn, vn = query_and_new(w)
    for b, g in units:
        check_unit(w, snap, res["scores"], res["sel"], res["cnt"], res["out"], res["lse"], q, kn, vn, b, g,
                   f"{what} b={b} g={g}", tail=tail)


def _pages_per_warp(res, ctas: int) -> int:
    """W of the attention kernel: selected pages of the batch over its 8 * ctas warps."""
    return -(-int(res["cnt"].sum()) // (8 * ctas))


def _default_ctas(w) -> int:
    """The attention grid without an override: one CTA per SM for a 16-bit-only cache, two
    per SM for a cache with quantised pools (at these batch sizes)."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    only16 = all(t == W.TIER_F16 for b in range(w.B) for t in w.tiers(b))
    return sms * (1 if only16 else 2)


@pytest.mark.parametrize("name, n_units", [("c1", 8), ("c2", 8), ("c3", 8), ("c4", 12)])
def test_full_size_four_calls_match_oracle(kvq, name, n_units):
    w = W.make(name)
    cache = kvq.cache_from_workload(w)
    step = kvq.DecodeStep(w, cache)
    step.run()
    res = _results(step, w)
    assert cache.err_bits() == 0, hex(cache.err_bits())
    # the attention kernel's pages per warp at this size
    assert _pages_per_warp(res, _default_ctas(w)) >= 2
    _check_units(w, cache, res, sample_units(w, n_units, seed=1), f"{name} full")


@pytest.mark.parametrize("name, path", [("c1", "fused"), ("c4", "fused"), ("c2", "three"), ("c4", "three")])
def test_full_size_other_paths_match_oracle(kvq, name, path):
    """The one-launch fused step, and kvq_append_scores (its score sweep beside the append,
    the appended pages' tiles held back) + select + attention, at full size."""
    w = W.make(name)
    cache = kvq.cache_from_workload(w)
    step = kvq.DecodeStep(w, cache)
    step.run_fused() if path == "fused" else step.run_three()
    res = _results(step, w)
    assert cache.err_bits() == 0, hex(cache.err_bits())
    _check_units(w, cache, res, sample_units(w, 12 if name == "c4" else 8, seed=2), f"{name} full {path}",
                 tail=path != "fused")


@pytest.mark.parametrize("name, cov, n_units", [("c1", 0.95, 6), ("c4", 0.9, 4)])
def test_full_size_coverage_selection_matches_oracle(kvq, name, cov, n_units):
    """Full-size coverage (nucleus) selection instead of the budget: c1 at 0.95 (~91 % of
    the 2049 pages of every (sequence, kv head) chosen, ~1 GB streamed) and c4 at 0.9 (128
    ragged rows of 151-4052 pages, four tiers).  Sampled units (c4's longest and shortest
    among them): the chosen set is the oracle's wherever its margin is clear, and every
    head's output is the oracle's attention over the set chosen."""
    from oracle.select import coverage_margin, forced_pages, select_coverage
    from tests.parity_helpers import check_output, oracle_step
    w = W.make(name)
    cache = kvq.cache_from_workload(w)
    step = kvq.DecodeStep(w, cache, coverage=cov)
    step.run()
    res = _results(step, w)
    assert cache.err_bits() == 0, hex(cache.err_bits())
    q, kn, vn = query_and_new(w)
    for b, g in sample_units(w, n_units, seed=4):
        sh = prepare(w, b, g)
        r0 = oracle_step(w, prepare(w, b, g), b, g, q, kn, vn)
        L, P = int(w.final_lens()[b]), r0["P"]
        got = res["sel"][b, g, :res["cnt"][b, g]]
        if coverage_margin(r0["scores"], P, L, w.sm_scale, cov, w.n_sink, w.n_recent) > 1e-4:
            want = select_coverage(r0["scores"], P, L, w.sm_scale, cov, w.n_sink, w.n_recent)
            assert list(got) == list(want), (b, g)
        assert forced_pages(P, w.n_sink, w.n_recent) <= set(got.tolist())
        r = oracle_step(w, sh, b, g, q, kn, vn, sel=got.astype(np.int64))
        for i in range(w.G):
            check_output(res["out"][b, g * w.G + i], r["out"][i], f"{name} coverage b={b} g={g}", w.dtype)


DEEP = {
    "c1_16bit": lambda: W.small("c1"),
    "alltiers_g1": lambda: W.make("c1", B=2, Hq=8, Hkv=8, lens=np.array([700, 333]), tier_fracs=ALL_TIERS,
                                  k_frac_bp=2000),
    "c4_ragged": lambda: W.small("c4"),
}


@pytest.mark.parametrize("ctas", [1, 2, 3, 7])
@pytest.mark.parametrize("name", list(DEEP))
def test_deep_pipeline_small_grid_matches_oracle(kvq, name, ctas):
    """Every unit of a small batch with the attention run on `ctas` CTAs: 2 to 24 pages per
    warp, segments that start and end mid-warp and span CTAs."""
    w = DEEP[name]()
    kvq.kvq_set_grid_override(ctas)
    try:
        cache = kvq.cache_from_workload(w)
        step = kvq.DecodeStep(w, cache)       # workspace sized for the overridden grid
        step.run()
        res = _results(step, w)
    finally:
        kvq.kvq_set_grid_override(0)
    assert cache.err_bits() == 0, hex(cache.err_bits())
    assert _pages_per_warp(res, ctas) >= 2
    _check_units(w, cache, res, [(b, g) for b in range(w.B) for g in range(w.Hkv)], f"{name} ctas={ctas}")


@pytest.mark.parametrize("ctas", [1, 5])
def test_deep_pipeline_fused_step_small_grid(kvq, ctas):
    w = W.small("c1")
    kvq.kvq_set_grid_override(ctas)
    try:
        cache = kvq.cache_from_workload(w)
        step = kvq.DecodeStep(w, cache)
        step.run_fused()
        res = _results(step, w)
    finally:
        kvq.kvq_set_grid_override(0)
    assert cache.err_bits() == 0, hex(cache.err_bits())
    _check_units(w, cache, res, [(b, g) for b in range(w.B) for g in range(w.Hkv)], f"fused ctas={ctas}",
                 tail=False)


@pytest.mark.parametrize("tiers", [None, ALL_TIERS], ids=["16bit", "alltiers"])
def test_every_page_selected_default_grid(kvq, tiers):
    """k = 100 %: 4 x 8 x 513 pages over the default grid: 14 pages per warp in 16-bit (one
    CTA per SM), 7 with quantised pools (two per SM)."""
    over = dict(B=4, lens=np.full(4, 8192), k_frac_bp=10000)
    if tiers:
        over["tier_fracs"] = tiers
    w = W.make("c1", **over)
    cache = kvq.cache_from_workload(w)
    step = kvq.DecodeStep(w, cache)
    step.run()
    res = _results(step, w)
    assert cache.err_bits() == 0, hex(cache.err_bits())
    assert _pages_per_warp(res, _default_ctas(w)) >= 7
    assert np.all(res["cnt"] == 513)
    _check_units(w, cache, res, sample_units(w, 12, seed=3), "all pages")


def _score_items_total(w) -> int:
    """Score items of kvq_decode_step's work queue: per (b, kv head), one item per 32 ring
    slots of 8 KB of page summaries (at least one)."""
    per_slot = 8192 // (2 * w.D)
    total = 0
    for b in range(w.B):
        P = w.pages_after(b)
        nsl = -(-P // per_slot)
        total += max(1, -(-nsl // 32)) * w.Hkv
    return total


def test_bounded_wait_runs_out_and_workspace_recovers(kvq):
    from sparse_mixed_precision_kvq_b200.kvq import DERR_TIMEOUT, WS_WAIT_LIMIT_WORD
    w = W.small("c1")
    cache = kvq.cache_from_workload(w)
    step = kvq.DecodeStep(w, cache)
    pre = snapshot(cache)
    words = step.ws.view(torch.int32)
    words[WS_WAIT_LIMIT_WORD] = 1000                 # 1 ms
    words[0] = _score_items_total(w)                 # the queue starts at the first attention item
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    step.run_fused()
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert cache.err_bits() & DERR_TIMEOUT, hex(cache.err_bits())
    assert dt < 1.0, dt                              # the 1 ms limit, not the 2 s default
    # nothing of the cache was touched: no score item ran, so no token was appended
    post = snapshot(cache)
    for t in range(6):
        if pre["pools"][t] is not None:
            assert np.array_equal(pre["pools"][t], post["pools"][t])
    assert np.array_equal(pre["summary"], post["summary"]) and np.array_equal(pre["ksum"], post["ksum"])
    # the same workspace, re-initialised, gives a correct step
    cache.err.zero_()
    kvq.kvq_workspace_init(step.ws)
    step.run_fused()
    res = _results(step, w)
    assert cache.err_bits() == 0, hex(cache.err_bits())
    assert int(step.ws.view(torch.int32)[WS_WAIT_LIMIT_WORD].item()) == 0
    _check_units(w, cache, res, [(b, g) for b in range(w.B) for g in range(w.Hkv)], "after timeout", tail=False)
    for b, g in [(0, 0), (w.B - 1, w.Hkv - 1)]:
        sh = prepare(w, b, g)
        check_pages(pre, sh, w, b, g, range(sh.P))
        check_summary(pre, sh, b, g, sh.P)
