"""One decode step of one layer for chosen (sequence, kv head) pairs.

Test infrastructure only (see ``oracle/__init__.py``).

The step follows the order the pages describe for a decode step (AMASS, "What is in
the box"; ARGUS, "The One-Minute Explanation"): the new token is written into its
page (quantised to the page's tier) and the page summary refreshed; every page is
scored from its summary; the top pages plus the forced sink/recent pages are
selected; attention runs over the selected pages with dequantisation on read.
Building the prefilled cache (``prepare``) is separate from the step itself.
"""
from __future__ import annotations

import numpy as np

from .attention import attend, token_index
from .cache import SeqHead, append, build
from .fp import bits16_to_f64
from .quad import quad_scores
from .score import page_scores
from .select import select


def prepare(w, b: int, g: int) -> SeqHead:
    """Build the prefilled cache of (sequence b, kv head g) of workload ``w``."""
    return build(w.keys_bits(b, g), w.values_bits(b, g), w.dtype, w.tiers(b),
                 capacity_pages=w.max_pages)


def step_pair(w, sh: SeqHead, b: int, g: int, q: np.ndarray, k_new=None, v_new=None,
              sel=None, quad=None) -> dict:
    """Run the step for one (b, g) on a prepared cache (mutated by the append).

    ``q`` is the fp64 query ``[Hq, D]`` of sequence b.  ``sel`` (optional) replaces
    the selection by a given page list, for testing attention on its own.  ``quad``
    (optional, an ``oracle.quad.QuadState`` of the same pair) switches the page score
    to the quad score; the append then also advances its state.
    """
    if w.append:
        pos = int(w.lens[b])
        append(sh, pos, k_new, v_new)
        if quad is not None:
            quad.append(pos, sh.korig[pos])
    P = sh.P
    G = w.G
    qg = q[g * G:(g + 1) * G]
    if quad is None:
        scores = page_scores(qg, sh.summary, P, w.max_pages)
    else:
        scores = quad_scores(qg, sh.summary, quad.lam, quad.basis, w.sm_scale, P, w.max_pages)
    chosen = select(scores, P, w.k_abs, w.k_frac_bp, w.n_sink, w.n_recent)
    use = chosen if sel is None else np.asarray(sel, dtype=np.int64)
    idx = token_index(use, sh.L)
    out = np.zeros((G, w.D))
    lse = np.zeros(G)
    for i in range(G):
        o, l, _, _ = attend(qg[i], sh.khat[idx], sh.vhat[idx], w.sm_scale)
        out[i], lse[i] = o, l
    return dict(scores=scores, sel=chosen, used=use, out=out, lse=lse, P=P, L=sh.L)


def decode_step(w, pairs=None) -> dict:
    """The whole step for the listed (b, g) pairs (all pairs by default)."""
    if pairs is None:
        pairs = [(b, g) for b in range(w.B) for g in range(w.Hkv)]
    q = bits16_to_f64(w.query_bits(), w.dtype)
    kn, vn = w.new_kv_bits() if w.append else (None, None)
    res = {}
    for b, g in pairs:
        sh = prepare(w, b, g)
        r = step_pair(w, sh, b, g, q[b],
                      None if kn is None else kn[b, g], None if vn is None else vn[b, g])
        r["cache"] = sh
        res[(b, g)] = r
    return res
