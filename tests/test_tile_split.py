"""The page-score sweeps' division of 16-page tiles among warps (csrc/tile_split.cuh),
restated on the host and checked on ragged, empty and over-long rows: every tile that
holds pages is scored by exactly one warp, each item's row and tile are found by the
binary search and by the forward cursor alike, and every score of every row, up to
max_pages, is written exactly once (by a tile or by the -inf fill past the tiles).

Row bg of a sequence of length L has P = min(max(ceil(L / 16), 0), max_pages) pages and
ceil(P / 16) tiles; pre is the exclusive prefix of the tile counts over the B * Hkv rows;
warp gw of nw takes items [gw * pw, (gw + 1) * pw), pw = ceil(total / nw); a tile writes
the scores of its 16 pages below max_pages (-inf past P); the fill writes -inf from the
row's first page past its tiles to max_pages.
"""
import numpy as np
import pytest


def _rows(lens, Hkv, max_pages):
    P = np.minimum(np.maximum((np.asarray(lens, dtype=np.int64) + 15) // 16, 0), max_pages)
    P = np.repeat(P, Hkv)
    tiles = (P + 15) // 16
    pre = np.zeros(P.size + 1, dtype=np.int64)
    pre[1:] = np.cumsum(tiles)
    return P, tiles, pre


def _row_of_item(pre, BH, i):
    lo, hi = 0, BH - 1
    while lo < hi:
        mid = (lo + hi + 1) >> 1
        if pre[mid] <= i:
            lo = mid
        else:
            hi = mid - 1
    return lo


def _check(lens, Hkv, max_pages, nw):
    P, tiles, pre = _rows(lens, Hkv, max_pages)
    BH, total = P.size, int(pre[-1])
    pw = (total + nw - 1) // nw if total else 0
    seen = np.zeros(total, dtype=np.int64)
    written = np.zeros((BH, max_pages), dtype=np.int64)
    for gw in range(nw):
        i0 = min(total, gw * pw)
        i1 = min(total, i0 + pw)
        seen[i0:i1] += 1
        if i0 >= i1:
            continue
        cur = _row_of_item(pre, BH, i0)
        for i in range(i0, i1):
            while pre[cur + 1] <= i:  # the forward cursor
                cur += 1
            bg = _row_of_item(pre, BH, i)
            assert bg == cur and pre[bg] <= i < pre[bg + 1]
            tile = i - pre[bg]
            for p in range(tile * 16, tile * 16 + 16):
                if p < max_pages:
                    written[bg, p] += 1
    for bg in range(BH):  # the fill past each row's tiles
        written[bg, tiles[bg] * 16:] += 1
    assert total == 0 or (seen.min() == 1 and seen.max() == 1)
    assert written.min() == 1 and written.max() == 1


@pytest.mark.parametrize("nw", [1, 7, 2064, 2368])
def test_ragged_rows(nw):
    rng = np.random.default_rng(nw)
    for _ in range(30):
        B = int(rng.integers(1, 40))
        Hkv = int(rng.choice([1, 2, 8]))
        max_pages = int(rng.integers(1, 300))
        lens = rng.integers(-20, 16 * max_pages + 200, B)  # empty, partial, full and over-long rows
        _check(lens, Hkv, max_pages, nw)


def test_workload_shapes():
    from sparse_mixed_precision_kvq_b200 import workloads as W
    for name in ("c1", "c3", "c4"):
        w = W.make(name)
        _check(w.final_lens(), w.Hkv, w.max_pages, 2064)
