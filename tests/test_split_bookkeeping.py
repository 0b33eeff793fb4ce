"""The sparse attention's split-K bookkeeping, restated on the host and checked for every
input shape: the flat work split, the partial slots and the merge ranges.

The kernel (csrc/attn.cu) lays the selected pages of all (sequence, kv head) segments out
as one flat list (segment bg holds min(max(cnt[bg], 0), kmax) pages from off[bg]); warp u
of `nworkers = num_ctas * 8` takes pages [u*W, (u+1)*W), W = ceil(total / nworkers), and
CTA n the pages of its 8 warps, [n*cw, (n+1)*cw), cw = 8*W.  A warp writes the partial of
every segment it touches but its last to global warp slot u + bg (the last one too after a
timeout); a CTA writes its merged partial of a segment that other CTAs also touch to CTA
slot n + bg; the CTAs touching segment bg are n0 = off[bg] // cw .. n1 = (off[bg+1]-1) // cw,
and the last of them to count its arrival (the one that reads n1 - n0 as the old count)
merges slots n0 + bg .. n1 + bg.  The workspace holds nworkers + B*Hkv warp slots and
num_ctas + B*Hkv CTA slots.  These tests check, over random and edge-case counts, that
every page is covered once, that no two writers share a slot, that every slot is inside
the workspace, and that the merge ranges name exactly the writers.
"""
import numpy as np
import pytest

WARPS = 8


def _split(cnt, kmax, num_ctas):
    c = np.minimum(np.maximum(np.asarray(cnt, dtype=np.int64), 0), kmax)
    BH = c.size
    off = np.zeros(BH + 1, dtype=np.int64)
    off[1:] = np.cumsum(c)
    total = int(off[-1])
    nworkers = num_ctas * WARPS
    W = (total + nworkers - 1) // nworkers
    return c, off, total, nworkers, W


def _segments_touching(off, lo, hi):
    """Segments with at least one page in [lo, hi)."""
    return [bg for bg in range(off.size - 1) if off[bg] < off[bg + 1] and off[bg] < hi and off[bg + 1] > lo]


def _check(cnt, kmax, num_ctas):
    c, off, total, nworkers, W = _split(cnt, kmax, num_ctas)
    BH = c.size
    wslots, slots = nworkers + BH, num_ctas + BH
    # 1) every page is covered by exactly one warp
    seen = np.zeros(total, dtype=np.int64)
    warp_segs = {}
    for u in range(nworkers):
        f0 = min(total, u * W)
        f1 = min(total, f0 + W)
        seen[f0:f1] += 1
        warp_segs[u] = _segments_touching(off, f0, f1)
    assert total == 0 or seen.min() == 1 and seen.max() == 1
    # 2) warp slots u + bg: unique over every (warp, segment it touches), inside the workspace
    wused = [u + bg for u, segs in warp_segs.items() for bg in segs]
    assert len(wused) == len(set(wused))
    assert all(0 <= s < wslots for s in wused)
    if total == 0:
        return
    cw = WARPS * W
    cta_segs = {}
    for n in range(num_ctas):
        cta0 = min(total, n * cw)
        cta1 = min(total, cta0 + cw)
        cta_segs[n] = _segments_touching(off, cta0, cta1) if cta0 < cta1 else []
        wb = n * WARPS
        for bg in cta_segs[n]:
            # 4) the CTA's merge range names exactly its warps that touch the segment
            w0 = max(wb, off[bg] // W) - wb
            w1 = min(wb + WARPS - 1, (off[bg + 1] - 1) // W) - wb
            assert set(range(wb + w0, wb + w1 + 1)) == {u for u in range(wb, wb + WARPS) if bg in warp_segs[u]}
    used = []
    for bg in range(BH):
        if off[bg] == off[bg + 1]:
            continue
        n0, n1 = off[bg] // cw, (off[bg + 1] - 1) // cw
        # 5) the CTAs touching the segment are n0 .. n1, one arrival each
        assert {n for n, segs in cta_segs.items() if bg in segs} == set(range(n0, n1 + 1))
        if n0 != n1:
            used += [n + bg for n in range(n0, n1 + 1)]
    # 3) CTA slots n + bg: unique, inside the workspace, and the final merge reads only them
    assert len(used) == len(set(used))
    assert all(0 <= s < slots for s in used)


@pytest.mark.parametrize("num_ctas", [1, 2, 5, 37, 148, 296])
def test_random_counts(num_ctas):
    rng = np.random.default_rng(num_ctas)
    for _ in range(40):
        BH = int(rng.integers(1, 160))
        kind = rng.integers(0, 4)
        if kind == 0:
            cnt = rng.integers(0, 400, BH)                    # ragged
        elif kind == 1:
            cnt = np.full(BH, int(rng.integers(1, 300)))      # equal rows
        elif kind == 2:
            cnt = rng.integers(0, 3, BH) * rng.integers(0, 900, BH)  # many empty segments
        else:
            cnt = rng.integers(-5, 50, BH)                    # negative counts clamp to 0
        kmax = int(rng.integers(1, 1000))
        _check(cnt, kmax, num_ctas)


def test_edge_cases():
    _check([0], 10, 148)                    # nothing selected
    _check([1], 10, 148)                    # one page, most warps idle
    _check([5] * 64, 5, 1)                  # one CTA holds everything
    _check([108] * 64, 200, 148)            # c1's shape: 64 segments of 108 pages
    _check([210] * 64, 300, 296)            # c2's shape on 2 CTAs per SM
    _check([427] * 8, 500, 296)             # c3's shape: few long segments, many CTAs each
    _check([1000] * 3, 64, 148)             # counts above kmax are clamped
    _check([7, 0, 0, 9, 0, 1], 10, 1)       # empty segments between full ones
