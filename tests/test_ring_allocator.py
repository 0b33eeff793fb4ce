"""The attention kernel's per-warp page ring (csrc/attn.cu, `issue_more`), restated on the
host and checked on every tier mix: pages in flight never overlap in the ring, no page
straddles the ring's end, and the warp can always make progress.

Allocation: a page of `bytes` (its K and V chunks) goes after the last page issued, or to
the ring's start when it does not fit before the end, once the space it needs has been
consumed; up to kNBar pages are in flight; consuming a page frees everything before its
end.  When nothing is in flight the ring restarts at offset 0, so any page that fits the
ring at all can be issued: without that restart a 12 KB ring holding 8 KB pages can reach
a state where the next page waits for space that only an in-flight page would free, with
none in flight.  Chunk sizes come from the library (`kvq_chunk_bytes`).
"""
import random

import pytest

K_NBAR = 8
RINGS = (12288, 24576)   # bytes per warp: two CTAs per SM, one CTA per SM


def _chunk_bytes():
    from sparse_mixed_precision_kvq_b200 import kvq
    return {D: {t: kvq.kvq_chunk_bytes(t, D) for t in range(6)} for D in (64, 128)}


def _run(ring, page_bytes, restart=True):
    """Issue and consume the pages in order; False if the warp gets stuck."""
    issued = consumed = head = tail = 0
    inflight = {}            # page -> (start, end), monotonic byte counters
    n = len(page_bytes)
    while consumed < n:
        while issued - consumed < K_NBAR and issued < n:
            if restart and issued == consumed:
                head = tail = 0
            b = page_bytes[issued]
            start = head
            pos = head % ring
            if pos + b > ring:
                start += ring - pos
            if start + b - tail > ring:
                break        # no room yet
            s0 = start % ring
            assert s0 + b <= ring, "a page straddles the ring's end"
            for (a0, a1) in inflight.values():
                c0 = a0 % ring
                assert s0 + b <= c0 or c0 + (a1 - a0) <= s0, "pages in flight overlap"
            inflight[issued] = (start, start + b)
            head = start + b
            issued += 1
        if issued == consumed:
            return False     # nothing in flight and nothing issued
        tail = inflight.pop(consumed)[1]
        consumed += 1
    return True


@pytest.mark.parametrize("ring", RINGS)
@pytest.mark.parametrize("D", [64, 128])
def test_every_tier_mix_makes_progress(ring, D):
    cb = _chunk_bytes()[D]
    mixes = [[0], [1], [5], [0, 1, 2, 3], [0, 2, 3, 4], [0, 1, 2, 3, 4, 5], [0, 5], [4, 0]]
    rng = random.Random(ring + D)
    for _ in range(3000):
        mix = rng.choice(mixes)
        pages = [2 * cb[rng.choice(mix)] for _ in range(rng.randint(1, 40))]
        assert max(pages) <= ring    # every page (16-bit at D = 128: 8 KB) fits either ring
        assert _run(ring, pages)


def test_restart_is_needed_on_the_narrow_ring():
    """Without the restart some sequences of 16-bit and quantised pages get stuck on the
    12 KB ring (the reason the restart exists)."""
    cb = _chunk_bytes()[128]
    rng = random.Random(1)
    stuck = 0
    for _ in range(3000):
        pages = [2 * cb[rng.choice([0, 1, 2, 3])] for _ in range(rng.randint(1, 40))]
        stuck += not _run(12288, pages, restart=False)
        assert _run(12288, pages, restart=True)
    assert stuck > 0
