"""GPU path vs the CPU oracle on reduced workloads (every element compared).

Covers, per workload: stored page bytes after the bulk build (bit-exact), the page
summaries and open-page key sums (bit-exact), the appended token's page bytes and
summary (bit-exact), the page scores (fp32 accumulation bound), the selected pages
(bit-exact where the k-th margin exceeds 1e-5), and the attention outputs (max abs
<= 1e-2, rel L2 <= 5e-3) and log-sum-exp.  All calls go through the C ABI.
"""
import math

import numpy as np
import pytest
import torch

from oracle import cache as ocache
from oracle.step import prepare
from sparse_mixed_precision_kvq_b200 import workloads as W
from tests.parity_helpers import (check_output, check_pages, check_scores, check_selection, check_summary,
                                  check_unit, oracle_step, out_to_f64, query_and_new, snapshot)

pytestmark = pytest.mark.gpu

ALL_TIERS = {W.TIER_F16: 0.16, W.TIER_I8: 0.17, W.TIER_I4: 0.17, W.TIER_I2: 0.17, W.TIER_I1: 0.17, W.TIER_F8: 0.16}
VARIANTS = {
    "c0": lambda: W.small("c0"),
    "c0_alltiers_fp16_d64": lambda: W.make("c0", lens=np.array([1000]), append=True, tier_fracs=ALL_TIERS),
    "c1": lambda: W.small("c1"),
    "c2": lambda: W.small("c2"),
    "c3": lambda: W.small("c3"),
    "c4": lambda: W.small("c4"),
    "g1_alltiers": lambda: W.make("c1", B=2, Hq=8, Hkv=8, lens=np.array([700, 333]), tier_fracs=ALL_TIERS,
                                  k_frac_bp=2000),
    "g2_alltiers": lambda: W.make("c4", B=3, Hq=16, Hkv=8, lens=np.array([513, 64, 2047]), tier_fracs=ALL_TIERS),
}


@pytest.fixture(scope="module")
def kvq():
    from sparse_mixed_precision_kvq_b200 import kvq as k
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return k


def _run(kvq, w, fused=False):
    cache = kvq.cache_from_workload(w)
    pre = snapshot(cache)
    step = kvq.DecodeStep(w, cache)
    if fused == "two":
        step.run_two()
    elif fused == "three":
        step.run_three()
    elif fused:
        step.run_fused()
    else:
        step.run()
    torch.cuda.synchronize()
    post = snapshot(cache)
    return cache, step, pre, post


PATHS = ["calls", "fused", "two", "three"]


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("name", list(VARIANTS))
def test_step_matches_oracle(kvq, name, path):
    """The four calls, the two-launch kvq_score_select + attention, and the one-launch
    kvq_decode_step, against the oracle."""
    w = VARIANTS[name]()
    cache, step, pre, post = _run(kvq, w, fused={"calls": False, "fused": True, "two": "two", "three": "three"}[path])
    assert cache.err_bits() == 0, hex(cache.err_bits())
    q, kn, vn = query_and_new(w)
    scores = step.scores.cpu().numpy()
    sel = step.sel.cpu().numpy()
    cnt = step.cnt.cpu().numpy()
    out = out_to_f64(step.out, w.dtype)
    lse = step.lse.cpu().numpy()
    for b in range(w.B):
        for g in range(w.Hkv):
            sh = prepare(w, b, g)
            P0 = sh.P
            check_pages(pre, sh, w, b, g, range(P0))
            check_summary(pre, sh, b, g, P0)
            if int(w.lens[b]) % 16:
                assert np.array_equal(pre["ksum"][b, g], sh.ksum)
            # after the step: the appended page, summaries, scores, selection, every output
            check_unit(w, post, scores, sel, cnt, out, lse, q, kn, vn, b, g, name, pages=[], tail=path != "fused")


@pytest.mark.parametrize("name", ["c0_alltiers_fp16_d64", "g1_alltiers", "c4"])
def test_dequant_values_bit_exact(kvq, name):
    """The values read back from every tier equal the oracle's fp32(c*scale+zero) / +-m / 16-bit."""
    w = VARIANTS[name]()
    cache = kvq.cache_from_workload(w)
    out = torch.empty((w.Hkv, 2, 16, w.D), dtype=torch.float32, device="cuda")
    for b in range(min(w.B, 2)):
        shs = [prepare(w, b, g) for g in range(w.Hkv)]
        P = shs[0].P
        for p in range(P):
            kvq.kvq_dequant_page(cache, b, p, out)
            got = out.cpu().numpy().astype(np.float64)
            n = min(16, int(w.lens[b]) - 16 * p)
            for g in range(w.Hkv):
                s = slice(16 * p, 16 * p + n)
                assert np.array_equal(got[g, 0, :n], shs[g].khat[s]), (b, p, g)
                assert np.array_equal(got[g, 1, :n], shs[g].vhat[s]), (b, p, g)
    assert cache.err_bits() == 0


def test_select_isolated_ties_and_nans(kvq):
    """Given identical fp32 scores (many ties, NaNs), the GPU selection is the oracle's exactly."""
    from oracle.select import select
    rng = np.random.default_rng(5)
    w = W.make("c4", B=16, Hq=8, Hkv=2, lens=rng.integers(0, 1200, 16), append=False)
    cache = kvq.cache_from_workload(w)
    P_cap = w.max_pages
    sc = rng.integers(-4, 5, (w.B, w.Hkv, P_cap)).astype(np.float32)
    sc[rng.random(sc.shape) < 0.02] = np.nan
    sc[rng.random(sc.shape) < 0.02] = -0.0
    for params in [(-1, 800, 1, 4), (5, 0, 0, 0), (-1, 10000, 2, 2), (0, 0, 3, 0), (1000, 0, 1, 1)]:
        prm = kvq.SelectParams(*params)
        kmax = P_cap
        scores = torch.from_numpy(sc).cuda()
        selt = torch.full((w.B, w.Hkv, kmax), -7, dtype=torch.int32, device="cuda")
        cntt = torch.zeros((w.B, w.Hkv), dtype=torch.int32, device="cuda")
        cache.err.zero_()
        kvq.kvq_select_topk(cache, scores, prm, selt, cntt, kmax)
        got_s, got_c = selt.cpu().numpy(), cntt.cpu().numpy()
        for b in range(w.B):
            P = (int(w.lens[b]) + 15) // 16
            for g in range(w.Hkv):
                want = select(sc[b, g].astype(np.float64), P, *params)
                assert list(got_s[b, g, :got_c[b, g]]) == list(want), (params, b, g)
        nan_any = any(np.isnan(sc[b, g, :(int(w.lens[b]) + 15) // 16]).any() for b in range(w.B) for g in range(w.Hkv))
        assert bool(cache.err_bits() & kvq.DERR_NAN_SCORE) == nan_any


def test_select_few_long_rows(kvq):
    """Few long rows (the 1024-thread selection): ragged lengths with an empty row, a
    one-page row, a row shorter than a bitmap word and rows of 4100-8193 pages; integer
    scores with heavy ties (the radix path), NaNs, -0 and every budget form.  The
    selection is the oracle's exactly."""
    from oracle.select import select
    rng = np.random.default_rng(11)
    lens = np.array([0, 16, 16 * 20 + 3, 16 * 4100, 16 * 8193 - 5])
    w = W.make("c4", B=5, Hq=4, Hkv=2, lens=lens, append=False)
    cache = kvq.cache_from_workload(w)
    P_cap = w.max_pages
    sc = rng.integers(-4, 5, (w.B, w.Hkv, P_cap)).astype(np.float32)
    sc[3, 1] = rng.normal(0, 1, P_cap).astype(np.float32)  # spread-out values: the value bins
    sc[rng.random(sc.shape) < 0.02] = np.nan
    sc[rng.random(sc.shape) < 0.02] = -0.0
    for params in [(-1, 500, 1, 4), (-1, 800, 1, 4), (5, 0, 0, 0), (-1, 10000, 2, 2), (0, 0, 3, 0),
                   (1000, 0, 1, 1), (40, 0, 0, 0)]:
        prm = kvq.SelectParams(*params)
        kmax = P_cap
        selt = torch.full((w.B, w.Hkv, kmax), -7, dtype=torch.int32, device="cuda")
        cntt = torch.zeros((w.B, w.Hkv), dtype=torch.int32, device="cuda")
        cache.err.zero_()
        kvq.kvq_select_topk(cache, torch.from_numpy(sc).cuda(), prm, selt, cntt, kmax)
        got_s, got_c = selt.cpu().numpy(), cntt.cpu().numpy()
        for b in range(w.B):
            P = (int(w.lens[b]) + 15) // 16
            for g in range(w.Hkv):
                want = select(sc[b, g].astype(np.float64), P, *params)
                assert list(got_s[b, g, :got_c[b, g]]) == list(want), (params, b, g)
        assert not (cache.err_bits() & ~kvq.DERR_NAN_SCORE)


def test_select_kmax_truncation_flag(kvq):
    w = W.small("c1", append=False)
    cache = kvq.cache_from_workload(w)
    step = kvq.DecodeStep(w, cache)
    step.scores_()
    small = 7
    sel = torch.zeros((w.B, w.Hkv, small), dtype=torch.int32, device="cuda")
    cnt = torch.zeros((w.B, w.Hkv), dtype=torch.int32, device="cuda")
    kvq.kvq_select_topk(cache, step.scores, step.params, sel, cnt, small)
    assert int(cnt.max()) == small
    assert cache.err_bits() & kvq.DERR_KMAX


@pytest.mark.parametrize("name", ["c2", "c4", "c0_alltiers_fp16_d64"])
def test_attention_isolated_random_selection(kvq, name):
    """Attention over a given (random) page list equals the oracle's over the same list."""
    w = VARIANTS[name]()
    cache = kvq.cache_from_workload(w)
    step = kvq.DecodeStep(w, cache)
    step.append()
    rng = np.random.default_rng(11)
    q, kn, vn = query_and_new(w)
    lists = {}
    selh = np.zeros((w.B, w.Hkv, step.kmax), dtype=np.int32)
    cnth = np.zeros((w.B, w.Hkv), dtype=np.int32)
    for b in range(w.B):
        P = w.pages_after(b)
        for g in range(w.Hkv):
            n = int(rng.integers(0, min(P, step.kmax) + 1)) if P else 0
            s = np.sort(rng.choice(P, size=n, replace=False)) if n else np.zeros(0, np.int64)
            lists[(b, g)] = s
            selh[b, g, :n] = s
            cnth[b, g] = n
    step.sel.copy_(torch.from_numpy(selh))
    step.cnt.copy_(torch.from_numpy(cnth))
    step.attend()
    torch.cuda.synchronize()
    assert cache.err_bits() == 0
    out = out_to_f64(step.out, w.dtype)
    lse = step.lse.cpu().numpy()
    for b in range(w.B):
        for g in range(w.Hkv):
            sh = prepare(w, b, g)
            r = oracle_step(w, sh, b, g, q, kn, vn, sel=lists[(b, g)])
            for i in range(w.G):
                h = g * w.G + i
                if lists[(b, g)].size == 0:
                    assert np.all(out[b, h] == 0) and np.isneginf(lse[b, h])
                else:
                    check_output(out[b, h], r["out"][i], f"{name} b={b} h={h}", w.dtype)


@pytest.mark.parametrize("path", PATHS)
def test_edge_cases_empty_short_and_overlapping(kvq, path):
    """Empty sequences, P < k (everything selected), sink/recent overlap, a page-aligned
    append that opens a page, and a ragged last page."""
    w = W.make("c4", B=6, Hq=8, Hkv=2, lens=np.array([0, 1, 15, 16, 40, 200]), append=True,
               n_sink=3, n_recent=3, k_abs=2, tier_fracs=ALL_TIERS)
    cache, step, pre, post = _run(kvq, w, fused={"calls": False, "fused": True, "two": "two", "three": "three"}[path])
    assert cache.err_bits() == 0
    q, kn, vn = query_and_new(w)
    out = out_to_f64(step.out, w.dtype)
    sel, cnt = step.sel.cpu().numpy(), step.cnt.cpu().numpy()
    for b in range(w.B):
        for g in range(w.Hkv):
            sh = prepare(w, b, g)
            r = oracle_step(w, sh, b, g, q, kn, vn)
            assert list(sel[b, g, :cnt[b, g]]) == list(r["sel"])
            check_pages(post, sh, w, b, g, range(sh.P))
            for i in range(w.G):
                check_output(out[b, g * w.G + i], r["out"][i], f"edge b={b}", w.dtype)


@pytest.mark.parametrize("path", PATHS)
def test_empty_selection_gives_zero_output(kvq, path):
    w = W.make("c4", B=3, Hq=8, Hkv=2, lens=np.array([0, 35, 0]), append=False)
    cache, step, pre, post = _run(kvq, w, fused={"calls": False, "fused": True, "two": "two", "three": "three"}[path])
    out = step.out.float().cpu().numpy()
    lse = step.lse.cpu().numpy()
    assert np.all(out[0] == 0) and np.all(out[2] == 0)
    assert np.all(np.isneginf(lse[0])) and np.all(np.isneginf(lse[2]))
    assert np.all(np.isfinite(lse[1]))


def test_bad_block_table_entry_is_flagged_not_fatal(kvq):
    """A selected page whose block-table entry names a bad tier is skipped and flagged."""
    w = W.small("c1", append=False)
    cache, step, pre, post = _run(kvq, w)
    bt = cache.block_table.clone()
    p = int(step.sel[0, 0, 3].item())
    cache.block_table[0, p] = -1          # tier 7: invalid
    cache.err.zero_()
    step.attend()
    torch.cuda.synchronize()
    assert cache.err_bits() & kvq.DERR_BAD_PAGE
    assert torch.isfinite(step.out.float()).all()
    cache.block_table.copy_(bt)


def test_fp16_metadata_saturation_flag(kvq):
    """A token whose group range exceeds fp16 saturates scale/zero like the oracle and is flagged."""
    w = W.make("c4", B=1, Hq=8, Hkv=2, lens=np.array([20]), append=True,
               tier_fracs={W.TIER_I4: 1.0})
    cache = kvq.cache_from_workload(w)
    step = kvq.DecodeStep(w, cache)
    big = np.zeros((1, 2, 128), dtype=np.float32)
    big[0, :, 0], big[0, :, 1] = -3e5, 3e5
    bits = W.f32_to_bf16_bits(big)
    step.k_new.copy_(torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16))
    step.append()
    torch.cuda.synchronize()
    assert cache.err_bits() & kvq.DERR_FP16_RANGE
    sh = prepare(w, 0, 0)
    ocache.append(sh, 20, bits[0, 0], w.new_kv_bits()[1][0, 0])
    check_pages(snapshot(cache), sh, w, 0, 0, [1])


@pytest.mark.parametrize("name", ["c2", "c4", "g2_alltiers"])
def test_fused_step_equals_calls_and_is_deterministic(kvq, name):
    """kvq_decode_step gives the four calls' scores and pages bit for bit, outputs within
    the output tolerance, and the same bits on every repeat (the workspace counters are
    back at zero after each call)."""
    if name == "g2_alltiers":
        w_na = W.make("c4", B=3, Hq=16, Hkv=8, lens=np.array([513, 64, 2047]), tier_fracs=ALL_TIERS, append=False)
    else:
        w_na = W.small(name, append=False)
    cache = kvq.cache_from_workload(w_na)
    step = kvq.DecodeStep(w_na, cache)
    step.run()
    torch.cuda.synchronize()
    ref = [t.clone() for t in (step.scores, step.sel, step.cnt, step.out, step.lse)]
    outs = []
    for _ in range(3):
        step.scores.fill_(7.0)
        step.sel.fill_(-3)
        step.out.zero_()
        step.run_fused()
        torch.cuda.synchronize()
        outs.append(step.out.clone())
        cnt = step.cnt.cpu().numpy()
        assert torch.equal(step.cnt, ref[2])
        for b in range(w_na.B):
            P = (int(w_na.lens[b]) + 15) // 16
            for g in range(w_na.Hkv):
                assert torch.equal(step.scores[b, g, :P], ref[0][b, g, :P]), (b, g)
                assert torch.equal(step.sel[b, g, :cnt[b, g]], ref[1][b, g, :cnt[b, g]]), (b, g)
        check_output(out_to_f64(step.out, w_na.dtype), out_to_f64(ref[3], w_na.dtype), name, w_na.dtype)
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])
    assert cache.err_bits() == 0


def test_fused_step_kmax_truncation_flag(kvq):
    w = W.small("c1", append=False)
    cache = kvq.cache_from_workload(w)
    step = kvq.DecodeStep(w, cache)
    small = 7
    sel = torch.zeros((w.B, w.Hkv, small), dtype=torch.int32, device="cuda")
    ws = torch.zeros(kvq.kvq_step_workspace_size(cache, small) // 4 + 4, dtype=torch.float32, device="cuda")
    kvq.kvq_decode_step(cache, None, None, None, step.q, step.params, step.scores, sel, step.cnt, small,
                        w.sm_scale, step.out, step.lse, ws)
    torch.cuda.synchronize()
    assert int(step.cnt.max()) == small
    assert cache.err_bits() & kvq.DERR_KMAX
    assert torch.isfinite(step.out.float()).all()


@pytest.mark.parametrize("P_cap", [3000, 5000])
def test_select_special_values_and_wide_ranges(kvq, P_cap):
    """Infinite scores, a range near the fp32 limit, all-equal scores, denormals and a
    large random batch: the selection is the oracle's exactly (ties on page index).
    5000 pages for 24 (b, kv head) pairs runs the 1024-thread selection."""
    from oracle.select import select
    rng = np.random.default_rng(7)
    B, Hkv = 12, 2
    w = W.make("c4", B=B, Hq=8, Hkv=Hkv, lens=np.full(B, 16 * P_cap), append=False)
    cache = kvq.cache_from_workload(w)
    sc = rng.normal(0, 3, (B, Hkv, w.max_pages)).astype(np.float32)
    sc[0, 0, rng.integers(0, P_cap, 20)] = np.inf
    sc[0, 1, rng.integers(0, P_cap, 20)] = -np.inf
    sc[1, 0] = rng.choice([-3e38, 3e38, 1.0, -1.0], w.max_pages).astype(np.float32)
    sc[1, 1] = 2.5
    sc[2, 0] = (rng.integers(-3, 4, w.max_pages) * 1e-42).astype(np.float32)   # denormals and zeros
    sc[2, 1] = rng.integers(0, 3, w.max_pages).astype(np.float32)              # three values only
    sc[3, 0, ::7] = np.nan
    for params in [(-1, 500, 1, 4), (-1, 9000, 0, 0), (37, 0, 2, 3)]:
        prm = kvq.SelectParams(*params)
        kmax = w.max_pages
        scores = torch.from_numpy(sc).cuda()
        selt = torch.full((B, Hkv, kmax), -7, dtype=torch.int32, device="cuda")
        cntt = torch.zeros((B, Hkv), dtype=torch.int32, device="cuda")
        kvq.kvq_select_topk(cache, scores, prm, selt, cntt, kmax)
        got_s, got_c = selt.cpu().numpy(), cntt.cpu().numpy()
        P = (int(w.lens[0]) + 15) // 16
        for b in range(B):
            for g in range(Hkv):
                want = select(sc[b, g].astype(np.float64), P, *params)
                assert list(got_s[b, g, :got_c[b, g]]) == list(want), (params, b, g)


@pytest.mark.parametrize("path", PATHS)
def test_long_context_many_pages(kvq, path):
    """A sequence of 8193 pages (131072 tokens + 1, as in the long-context workload): the
    selection keeps all of its keys on chip; pages, selection and output as the oracle's."""
    w = W.make("c3", lens=np.array([131072]), Hq=8, Hkv=2)
    cache, step, pre, post = _run(kvq, w, fused={"calls": False, "fused": True, "two": "two", "three": "three"}[path])
    assert cache.err_bits() == 0, hex(cache.err_bits())
    q, kn, vn = query_and_new(w)
    sel, cnt = step.sel.cpu().numpy(), step.cnt.cpu().numpy()
    out = out_to_f64(step.out, w.dtype)
    for g in range(w.Hkv):
        sh = prepare(w, 0, g)
        r = oracle_step(w, sh, 0, g, q, kn, vn)
        assert check_selection(sel[0, g, :cnt[0, g]], r["sel"], r["scores"], w, r["P"])
        for i in range(w.G):
            check_output(out[0, g * w.G + i], r["out"][i], f"long g={g}", w.dtype)


@pytest.mark.parametrize("name", ["c1", "c4", "g2_alltiers"])
def test_score_select_equals_calls(kvq, name):
    """kvq_score_select (append + scores + selection in one launch) and kvq_append_scores
    leave the same cache bytes, scores, selection and (through the same attention call)
    outputs as the four calls."""
    w = VARIANTS[name]()
    outs = []
    for how in ("calls", "two", "three"):
        cache = kvq.cache_from_workload(w)
        step = kvq.DecodeStep(w, cache)
        {"calls": step.run, "two": step.run_two, "three": step.run_three}[how]()
        torch.cuda.synchronize()
        outs.append((snapshot(cache), step.scores.clone(), step.sel.clone(), step.cnt.clone(), step.out.clone()))
        assert cache.err_bits() == 0, hex(cache.err_bits())
    (s0, sc0, sel0, cnt0, o0) = outs[0]
    for (s1, sc1, sel1, cnt1, o1) in outs[1:]:
        for t, (p0, p1) in enumerate(zip(s0["pools"], s1["pools"])):
            assert (p0 is None) == (p1 is None) and (p0 is None or np.array_equal(p0, p1)), t
        for k in ("bt", "summary", "ksum"):
            assert np.array_equal(s0[k], s1[k]), k
        assert torch.equal(sc0, sc1) and torch.equal(cnt0, cnt1) and torch.equal(o0, o1)
        c = cnt0.cpu().numpy()
        for b in range(w.B):
            for g in range(w.Hkv):
                assert torch.equal(sel0[b, g, :c[b, g]], sel1[b, g, :c[b, g]])


@pytest.mark.parametrize("tiers", [None, ALL_TIERS])
def test_append_scores_two_steps_equal_calls(kvq, tiers):
    """Two decode steps back to back (the second append chained right after the first
    step's attention, one sequence skipped, appended pages at a page start, mid-page and a
    page end): kvq_append_scores, whose sweep scores the tiles without an appended page
    before the append completes, leaves the bytes, scores, selection and outputs of the
    four separate calls."""
    over = dict(B=5, Hq=16, Hkv=2, lens=np.array([100, 47, 512, 1000, 40]))
    if tiers is not None:
        over["tier_fracs"] = tiers
    w = W.make("c4", **over)
    outs = []
    for how in ("calls", "three"):
        cache = kvq.cache_from_workload(w)
        step = kvq.DecodeStep(w, cache)
        run = step.run if how == "calls" else step.run_three
        run()
        step.pos += 1
        step.pos[1] = -1
        cache.seq_len += 1
        cache.seq_len[1] -= 1
        step.k_new.mul_(-0.5)
        run()
        torch.cuda.synchronize()
        assert cache.err_bits() == 0, hex(cache.err_bits())
        outs.append((snapshot(cache), step.scores.clone(), step.sel.clone(), step.cnt.clone(), step.out.clone()))
    (s0, sc0, sel0, cnt0, o0), (s1, sc1, sel1, cnt1, o1) = outs
    for t, (p0, p1) in enumerate(zip(s0["pools"], s1["pools"])):
        assert (p0 is None) == (p1 is None) and (p0 is None or np.array_equal(p0, p1)), t
    for k in ("bt", "summary", "ksum"):
        assert np.array_equal(s0[k], s1[k]), k
    assert torch.equal(sc0, sc1) and torch.equal(cnt0, cnt1) and torch.equal(o0, o1)
    c = cnt0.cpu().numpy()
    for b in range(w.B):
        for g in range(w.Hkv):
            assert torch.equal(sel0[b, g, :c[b, g]], sel1[b, g, :c[b, g]])


@pytest.mark.parametrize("B,Hkv", [(1600, 8), (300, 8)])
def test_ragged_scores_both_splits(kvq, B, Hkv):
    """kvq_page_scores on a ragged batch with empty sequences: with 12,800 (sequence, kv
    head) rows the sweep divides whole max_pages rows among the warps, with 2,400 it
    divides only the tiles that hold pages (and fills -inf past each length).  Scores of a
    sample of units, the empty ones included, against the oracle's."""
    rng = np.random.default_rng(B)
    lens = rng.integers(0, 400, B)
    lens[:4] = [0, 1, 16, 399]
    lens[-1] = 0
    w = W.make("c4", B=B, Hq=Hkv, Hkv=Hkv, lens=lens, append=False)
    cache = kvq.cache_from_workload(w)
    step = kvq.DecodeStep(w, cache)
    step.scores_()
    torch.cuda.synchronize()
    assert cache.err_bits() == 0, hex(cache.err_bits())
    scores = step.scores.cpu().numpy()
    q, kn, vn = query_and_new(w)
    units = {(0, 0), (1, Hkv - 1), (2, 3), (3, 5), (B - 1, Hkv - 1), (B - 1, 0)}
    units |= {(int(b), int(g)) for b, g in zip(rng.integers(0, B, 6), rng.integers(0, Hkv, 6))}
    for b, g in sorted(units):
        sh = prepare(w, b, g)
        r = oracle_step(w, sh, b, g, q, kn, vn)
        check_scores(scores[b, g], r["scores"], q[b, g:g + 1], sh.summary, r["P"])


@pytest.mark.parametrize("P_cap", [700, 5000])
def test_coverage_selection_matches_oracle(kvq, P_cap):
    """Coverage (nucleus) selection: the GPU set is the oracle's wherever the cut is not
    within rounding of another decision (ties, NaNs, partial last pages, every coverage)."""
    from oracle.select import coverage_margin, select_coverage
    rng = np.random.default_rng(P_cap)
    B, Hkv = 12, 2
    lens = rng.integers(1, 16 * P_cap + 1, B)
    lens[0] = 16 * P_cap
    w = W.make("c4", B=B, Hq=8, Hkv=Hkv, lens=lens, append=False)
    cache = kvq.cache_from_workload(w)
    sc = rng.normal(0, 3, (B, Hkv, w.max_pages)).astype(np.float32)
    sc[1] = np.round(sc[1])           # ties
    sc[2, 0, ::5] = np.nan
    sc[3] = 1.5                       # every page the same score
    checked = 0
    for cov, scale, ns, nr in [(0.95, 0.088, 1, 4), (0.5, 0.3, 0, 0), (0.99, 0.05, 2, 1), (1.0, 1.0, 0, 2),
                               (0.9, 0.088, 0, 0)]:
        prm = kvq.SelectParams(-1, 0, ns, nr, int(round(cov * 1e6)), scale)
        kmax = w.max_pages
        selt = torch.full((B, Hkv, kmax), -7, dtype=torch.int32, device="cuda")
        cntt = torch.zeros((B, Hkv), dtype=torch.int32, device="cuda")
        cache.err.zero_()
        kvq.kvq_select_topk(cache, torch.from_numpy(sc).cuda(), prm, selt, cntt, kmax)
        got_s, got_c = selt.cpu().numpy(), cntt.cpu().numpy()
        for b in range(B):
            L = int(w.lens[b])
            P = (L + 15) // 16
            for g in range(Hkv):
                want = select_coverage(sc[b, g].astype(np.float64), P, L, scale, int(round(cov * 1e6)) * 1e-6, ns, nr)
                got = list(got_s[b, g, :got_c[b, g]])
                if coverage_margin(sc[b, g].astype(np.float64), P, L, scale, cov, ns, nr) > 1e-5:
                    assert got == list(want), (cov, scale, b, g, len(got), len(want))
                    checked += 1
                else:
                    assert abs(len(got) - len(want)) <= 1
        assert not (cache.err_bits() & ~kvq.DERR_NAN_SCORE)
    assert checked >= 40


@pytest.mark.parametrize("kind", ["ties", "wide"])
def test_coverage_exact_ties_and_wide_masses(kvq, kind):
    """Coverage selection where the cut lands inside a group of exactly equal masses
    (scores from four values: the group's lowest pages are taken, as many as reach the
    target) or where the masses span hundreds of binades (the search descends through many
    digit passes).  The set must be the oracle's wherever the covered mass is not within
    1e-5 of the target; exact ties are part of the rule, not an ambiguity."""
    from oracle.select import forced_pages, page_masses, select_coverage
    import math
    rng = np.random.default_rng(11 if kind == "ties" else 12)
    B, Hkv = 8, 2
    lens = rng.integers(200, 16 * 600 + 1, B)
    w = W.make("c4", B=B, Hq=8, Hkv=Hkv, lens=lens, append=False)
    cache = kvq.cache_from_workload(w)
    if kind == "ties":
        sc = (rng.integers(0, 4, (B, Hkv, w.max_pages)) * 2.0).astype(np.float32)
        cases = [(0.3, 1.0, 1, 2), (0.5, 1.0, 0, 0), (0.7, 0.7, 2, 1), (0.9, 1.0, 0, 3), (0.97, 0.5, 1, 0)]
    else:
        sc = rng.normal(0, 40, (B, Hkv, w.max_pages)).astype(np.float32)
        cases = [(0.999, 1.0, 1, 2), (0.9999, 0.5, 0, 0), (0.5, 2.0, 0, 1), (0.99, 0.25, 2, 0)]
    checked = 0
    for cov, scale, ns, nr in cases:
        ppm = int(round(cov * 1e6))
        prm = kvq.SelectParams(-1, 0, ns, nr, ppm, scale)
        kmax = w.max_pages
        selt = torch.full((B, Hkv, kmax), -7, dtype=torch.int32, device="cuda")
        cntt = torch.zeros((B, Hkv), dtype=torch.int32, device="cuda")
        cache.err.zero_()
        kvq.kvq_select_topk(cache, torch.from_numpy(sc).cuda(), prm, selt, cntt, kmax)
        got_s, got_c = selt.cpu().numpy(), cntt.cpu().numpy()
        assert cache.err_bits() == 0
        for b in range(B):
            L = int(w.lens[b])
            P = (L + 15) // 16
            for g in range(Hkv):
                s64 = sc[b, g].astype(np.float64)
                want = select_coverage(s64, P, L, scale, ppm * 1e-6, ns, nr)
                got = list(got_s[b, g, :got_c[b, g]])
                # distance of the covered mass from the target, before and after the last page
                m = page_masses(s64, P, L, scale)
                F = forced_pages(P, ns, nr)
                total, target = math.fsum(m), ppm * 1e-6 * math.fsum(m)
                covered = math.fsum(m[p] for p in F)
                order = sorted((p for p in range(P) if p not in F), key=lambda p: (-m[p], p))
                k = 0
                while k < len(order) and covered < target:
                    covered += m[order[k]]
                    k += 1
                before = covered - (m[order[k - 1]] if k else 0.0)
                dist = min(abs(target - before), abs(covered - target)) / total
                gap_ok = not (0 < k < len(order)) or m[order[k - 1]] == m[order[k]] or \
                    (m[order[k - 1]] - m[order[k]]) / m[order[k - 1]] > 1e-5
                if dist > 1e-5 and gap_ok:
                    assert got == list(want), (kind, cov, b, g, len(got), len(want))
                    checked += 1
    assert checked >= 40


def test_coverage_step_through_attention(kvq):
    """A whole step with coverage selection: the pages chosen and the attention over them
    match the oracle's."""
    from oracle.select import coverage_margin, select_coverage
    w = W.small("c1")
    cache = kvq.cache_from_workload(w)
    step = kvq.DecodeStep(w, cache)
    step.params = kvq.SelectParams(-1, 0, w.n_sink, w.n_recent, 900000, w.sm_scale)
    step.kmax = w.max_pages
    step.sel = torch.zeros((w.B, w.Hkv, step.kmax), dtype=torch.int32, device="cuda")
    step.ws = torch.zeros(max(kvq.kvq_workspace_size(cache, step.kmax), 1 << 16) // 4 + 4, dtype=torch.float32,
                          device="cuda")
    step.run()
    torch.cuda.synchronize()
    assert cache.err_bits() == 0, hex(cache.err_bits())
    q, kn, vn = query_and_new(w)
    sel, cnt = step.sel.cpu().numpy(), step.cnt.cpu().numpy()
    out = out_to_f64(step.out, w.dtype)
    scores = step.scores.cpu().numpy()
    for b in range(w.B):
        for g in range(w.Hkv):
            sh = prepare(w, b, g)
            r0 = oracle_step(w, prepare(w, b, g), b, g, q, kn, vn)
            L, P = int(w.final_lens()[b]), r0["P"]
            want = select_coverage(r0["scores"], P, L, w.sm_scale, 0.9, w.n_sink, w.n_recent)
            if coverage_margin(r0["scores"], P, L, w.sm_scale, 0.9, w.n_sink, w.n_recent) > 1e-4:
                assert list(sel[b, g, :cnt[b, g]]) == list(want)
            r = oracle_step(w, sh, b, g, q, kn, vn, sel=sel[b, g, :cnt[b, g]].astype(np.int64))
            for i in range(w.G):
                check_output(out[b, g * w.G + i], r["out"][i], f"coverage b={b}", w.dtype)
