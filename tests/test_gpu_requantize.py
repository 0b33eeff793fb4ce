"""Tier demotion on the GPU (kvq_requantize_pages) vs the oracle's ``requantize``.

Every page of every (sequence, kv head) is compared bit for bit after a seeded mix of
demotions (each page to a random lower tier, partial last pages included), then a whole
decode step (append into a demoted open page, scores, selection, attention) runs on the
demoted cache and is compared with the oracle's step on the demoted oracle cache.
"""
import numpy as np
import pytest
import torch

from oracle import cache as ocache
from oracle.step import prepare
from sparse_mixed_precision_kvq_b200 import workloads as W
from tests.parity_helpers import (check_output, check_pages, check_selection, oracle_step, out_to_f64,
                                  query_and_new, snapshot)

pytestmark = pytest.mark.gpu

ALL_TIERS = {W.TIER_F16: 0.16, W.TIER_I8: 0.17, W.TIER_I4: 0.17, W.TIER_I2: 0.17, W.TIER_I1: 0.17, W.TIER_F8: 0.16}
CASES = {
    "bf16_d128": lambda: W.make("c1", B=2, Hq=16, Hkv=4, lens=np.array([700, 333]), tier_fracs=ALL_TIERS,
                                k_frac_bp=2000),
    "f16_d64": lambda: W.make("c0", B=2, lens=np.array([1000, 77]), append=True, tier_fracs=ALL_TIERS),
}


@pytest.fixture(scope="module")
def kvq():
    from sparse_mixed_precision_kvq_b200 import kvq as k
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return k


CASCADE = [W.TIER_F16, W.TIER_F8, W.TIER_I8, W.TIER_I4, W.TIER_I2, W.TIER_I1]  # hot to cold


def demotion_plan(w, seed=7, frac=0.6):
    """(b, page, new tier) for a seeded subset of the prefilled pages, each to a colder tier
    of the cascade; the last prefilled page of every sequence is always in the plan (when
    it can move)."""
    rng = np.random.default_rng(seed)
    plan = []
    for b in range(w.B):
        tiers = w.tiers(b)
        P0 = w.pages_before(b)
        for p in range(P0):
            t = int(tiers[p])
            pos = CASCADE.index(t)
            if t == W.TIER_I1 or (p != P0 - 1 and rng.random() > frac):
                continue
            plan.append((b, p, CASCADE[int(rng.integers(pos + 1, len(CASCADE)))]))
    return plan


def apply_plan(kvq, w, plan):
    """Cache with spare slots, demoted on the GPU; returns (cache, items, new entries)."""
    spare = [0] * 6
    for _, _, t in plan:
        spare[t] += 1
    _, _, counts = w.slot_map()
    cache = kvq.cache_from_workload(w, spare=spare)
    nxt = list(counts)
    items = []
    for b, p, t in plan:
        items.append((b, p, int(np.uint32((t << 29) | nxt[t]).view(np.int32))))
        nxt[t] += 1
    it = torch.tensor(items, dtype=torch.int32, device="cuda")
    kvq.kvq_requantize_pages(cache, it)
    torch.cuda.synchronize()
    return cache, items


@pytest.mark.parametrize("name", sorted(CASES))
def test_requantized_pages_match_the_oracle(kvq, name):
    w = CASES[name]()
    plan = demotion_plan(w)
    assert len(plan) > 10
    cache, items = apply_plan(kvq, w, plan)
    assert cache.err_bits() == 0, hex(cache.err_bits())
    snap = snapshot(cache)
    for b, p, e in items:
        assert int(snap["bt"][b, p]) == e
    for b in range(w.B):
        for g in range(w.Hkv):
            sh = prepare(w, b, g)
            for bb, p, t in plan:
                if bb == b:
                    ocache.requantize(sh, p, t)
            check_pages(snap, sh, w, b, g, range(w.pages_before(b)))
            assert np.array_equal(snap["summary"][b, g, :sh.P], sh.summary_bits[:sh.P])


@pytest.mark.parametrize("name", sorted(CASES))
def test_decode_step_on_a_demoted_cache(kvq, name):
    w = CASES[name]()
    plan = demotion_plan(w, seed=11)
    cache, _ = apply_plan(kvq, w, plan)
    step = kvq.DecodeStep(w, cache)
    step.run()
    torch.cuda.synchronize()
    assert cache.err_bits() == 0, hex(cache.err_bits())
    snap = snapshot(cache)
    q, kn, vn = query_and_new(w)
    out = out_to_f64(step.out, w.dtype)
    sel, cnt = step.sel.cpu().numpy(), step.cnt.cpu().numpy()
    scores = step.scores.cpu().numpy()
    for b in range(w.B):
        for g in range(w.Hkv):
            sh = prepare(w, b, g)
            for bb, p, t in plan:
                if bb == b:
                    ocache.requantize(sh, p, t)
            r = oracle_step(w, sh, b, g, q, kn, vn)
            check_pages(snap, sh, w, b, g, range(sh.P))  # the append wrote into the demoted tier
            if not check_selection(sel[b, g, :cnt[b, g]], r["sel"], scores[b, g], w, sh.P):
                continue
            for i in range(w.G):
                check_output(out[b, g * w.G + i], r["out"][i], f"b={b} g={g} h={i}", w.dtype)


def test_invalid_items_are_skipped_with_an_error_bit(kvq):
    w = CASES["f16_d64"]()
    cache = kvq.cache_from_workload(w, spare=[0, 1, 1, 1, 1, 1])
    bt0 = cache.block_table.clone()
    pools0 = [None if p is None else p.clone() for p in cache.pools]
    _, _, counts = w.slot_map()
    e = int(bt0[0, 5].item()) & 0xFFFFFFFF
    tier, slot = e >> 29, e & 0x1FFFFFFF

    def ent(t, s):
        return int(np.uint32((t << 29) | s).view(np.int32))

    bad = [
        (0, 5, ent(tier, slot)),                   # its own slot
        (0, 5, ent(0, counts[0])),                 # the 16-bit tier is not a demotion target
        (0, 5, ent(2, counts[2] + 5)),             # slot past the pool
        (2, 0, ent(2, counts[2])),                 # sequence out of range
        (1, w.max_pages, ent(2, counts[2])),       # page out of range
        (1, 10, ent(2, counts[2])),                # a page holding no tokens (77 tokens: pages 0..4)
        (0, 3, ent(6, 0)),                         # no such tier
        (0, 3, ent(7, 0)),                         # no such tier
    ]
    kvq.kvq_requantize_pages(cache, torch.tensor(bad, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert cache.err_bits() == 0x1
    assert torch.equal(cache.block_table, bt0)
    for a, b0 in zip(cache.pools, pools0):
        assert (a is None) == (b0 is None) and (a is None or torch.equal(a, b0))
    cache.err.zero_()
    kvq.kvq_requantize_pages(cache, None)        # n == 0: nothing launched
    torch.cuda.synchronize()
    assert cache.err_bits() == 0 and torch.equal(cache.block_table, bt0)


def _tie_values(D, L, seed=3):
    """fp16 K/V rows [L, D] whose 32-channel groups put the exact quotients of the target
    tiers on rounding ties (x = k + 1/2 with lo = 0 and hi = 2^b - 1, so scale = 1 and
    zero = 0), mixed with random groups, signed zeros and constant groups."""
    rng = np.random.default_rng(seed)
    x = rng.normal(0, 2, (2, L, D))
    for t in range(L):
        qmax = (255, 15, 3)[(t // 16) % 3]
        for kind in range(2):
            g0 = x[kind, t, :32]
            g0[:] = (np.arange(32) % (qmax + 1)) + 0.5
            g0[g0 > qmax] = qmax
            g0[0], g0[1] = 0.0, qmax
            if t % 4 == 1:
                x[kind, t, 32:64] = 0.0
                x[kind, t, 32:64:3] = -0.0          # a constant group of mixed signed zeros
            if t % 4 == 2:
                x[kind, t, 32:40] = -0.0            # a zero minimum of either sign
                x[kind, t, 40:64] = np.abs(x[kind, t, 40:64])
    return x.astype(np.float16).view(np.uint16)


@pytest.mark.parametrize("D", [64, 128])
def test_requantize_rounding_ties_and_signed_zeros(kvq, D):
    """Pages 0-2 (16-bit) move to int8, int4, int2: every tie group takes the exact fp64
    route and rounds half to even; then int8 -> int2, int4 -> 1-bit, int2 -> fp8, and
    fp8 -> int4."""
    L, Hkv = 40, 2
    bits = [_tie_values(D, L, seed=g) for g in range(Hkv)]
    cache = kvq.PagedCache(1, 2 * Hkv, Hkv, D, 3, "f16", [3, 3, 3, 3, 3, 3], "cuda")
    cache.block_table.copy_(torch.from_numpy(kvq.encode_block_table(np.zeros((1, 3), np.int64),
                                                                    np.arange(3)[None])))
    cache.seq_len.fill_(L)
    k = torch.from_numpy(np.stack([b_[0] for b_ in bits]).view(np.int16)).cuda()
    v = torch.from_numpy(np.stack([b_[1] for b_ in bits]).view(np.int16)).cuda()
    kvq.kvq_build_pages(cache, k, v, torch.tensor([0, L], dtype=torch.int64, device="cuda"))

    def ent(t, s):
        return int(np.uint32((t << 29) | s).view(np.int32))

    heads = [ocache.build(b_[0], b_[1], "f16", np.zeros(3, np.int64)) for b_ in bits]
    for plan in ([(0, 1, 0), (1, 2, 0), (2, 3, 0)], [(0, 3, 1), (1, 4, 1), (2, 5, 0)], [(2, 2, 1)]):
        items = torch.tensor([(0, p, ent(t, s)) for p, t, s in plan], dtype=torch.int32, device="cuda")
        kvq.kvq_requantize_pages(cache, items)
        torch.cuda.synchronize()
        for sh in heads:
            for p, t, _ in plan:
                ocache.requantize(sh, p, t)
        assert cache.err_bits() == 0, hex(cache.err_bits())
        snap = snapshot(cache)
        for g, sh in enumerate(heads):
            check_pages(snap, sh, W.make("c0", Hq=2 * Hkv, Hkv=Hkv, D=D, lens=np.array([L])), 0, g, range(3))
