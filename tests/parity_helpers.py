"""Shared helpers for the GPU-vs-oracle parity tests (imported by tests, not collected)."""
from __future__ import annotations

import numpy as np

from oracle import cache as ocache
from oracle.attention import attend, token_index
from oracle.fp import bits16_to_f64
from oracle.layout import chunk_bytes
from oracle.select import kth_margin
from oracle.step import prepare, step_pair

# Output tolerance for bf16/fp16 attention outputs: max |gpu - oracle| <= 1e-2 and
# ||gpu - oracle||_2 / ||oracle||_2 <= 5e-3 (checked per (sequence, kv head) group).
ATOL_MAX = 1e-2
REL_L2 = 5e-3
# Selected sets must match wherever the k-th score margin exceeds this (relative).
MARGIN = 1e-5


def pools_to_cpu(cache):
    """Every pool's bytes; a tier with a separate V pool gives a (K pool, V pool) pair."""
    vpools = getattr(cache, "vpools", [None] * len(cache.pools))
    return [None if p is None else (p.cpu().numpy() if v is None else (p.cpu().numpy(), v.cpu().numpy()))
            for p, v in zip(cache.pools, vpools)]


def gpu_chunk(pools, bt: np.ndarray, Hkv: int, D: int, b: int, p: int, g: int, kind: int):
    e = int(bt[b, p]) & 0xFFFFFFFF
    tier, slot = e >> 29, e & 0x1FFFFFFF
    cb = chunk_bytes(tier, D)
    if isinstance(pools[tier], tuple):  # separate K and V pools
        o = (slot * Hkv + g) * cb
        return tier, pools[tier][kind][o:o + cb]
    o = ((slot * Hkv + g) * 2 + kind) * cb
    return tier, pools[tier][o:o + cb]


def snapshot(cache):
    return dict(pools=pools_to_cpu(cache), bt=cache.block_table.cpu().numpy(),
                summary=cache.summary.cpu().numpy().view(np.uint16),
                ksum=cache.open_ksum.cpu().numpy())


def check_pages(snap, sh, w, b, g, pages):
    """Chunk bytes of the listed pages, bit for bit."""
    for p in pages:
        for kind, kk in ((0, "k"), (1, "v")):
            tier, got = gpu_chunk(snap["pools"], snap["bt"], w.Hkv, w.D, b, p, g, kind)
            want = ocache.page_bytes(sh, p, kk)
            assert tier == int(sh.tiers[p])
            if not np.array_equal(got, want):
                bad = np.nonzero(got != want)[0]
                raise AssertionError(f"b={b} g={g} page={p} kind={kk} tier={tier}: {bad.size} bytes differ, "
                                     f"first at {bad[:8]}")


def check_summary(snap, sh, b, g, P):
    got = snap["summary"][b, g, :P]
    want = sh.summary_bits[:P]
    assert np.array_equal(got, want), f"summary differs at pages {np.nonzero((got != want).any(1))[0][:8]}"


def check_scores(gpu_scores: np.ndarray, ref: np.ndarray, q_group: np.ndarray, summary: np.ndarray, P: int,
                 tail: bool = True):
    """fp32 scores within the fp32 accumulation bound of the fp64 oracle's (and -inf past
    the last page when ``tail``: kvq_page_scores writes them, kvq_decode_step does not)."""
    if tail:
        assert np.all(np.isneginf(gpu_scores[P:]))
    if P == 0:
        return
    mag = (np.abs(summary[:P]) @ np.abs(q_group).T).max(1)
    err = np.abs(gpu_scores[:P].astype(np.float64) - ref[:P])
    assert np.all(err <= 2e-6 * mag + 1e-30), f"max score error {err.max()}"


def check_selection(gpu_sel: np.ndarray, ref_sel: np.ndarray, scores: np.ndarray, w, P: int) -> bool:
    """Sets must be equal when the k-th margin is > MARGIN; returns whether they are equal."""
    same = np.array_equal(np.sort(gpu_sel), ref_sel)
    if not same:
        m = kth_margin(scores, P, w.k_abs, w.k_frac_bp, w.n_sink, w.n_recent)
        assert m <= MARGIN, f"selection differs with margin {m}"
    assert np.all(np.diff(gpu_sel) > 0), "selection not ascending"
    return same


def out_ulp(ref: np.ndarray, dtype: str) -> np.ndarray:
    """One unit in the last place of the output dtype at |ref| (normal range)."""
    mant = 7 if dtype == "bf16" else 10
    e = np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -14)))
    return 2.0 ** (e - mant)


def check_output(gpu: np.ndarray, ref: np.ndarray, what="", dtype="bf16"):
    """max |gpu - ref| <= 1e-2 (or one output-dtype ulp where that is larger: a bf16 value
    of magnitude >= 4 cannot be rounded to within 1e-2), and rel L2 <= 5e-3."""
    err = np.abs(gpu - ref)
    rel = np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-30)
    bound = np.maximum(ATOL_MAX, out_ulp(ref, dtype))
    assert np.all(err <= bound), f"{what}: max abs err {err.max()} (bound {bound[np.argmax(err - bound)]})"
    assert rel <= REL_L2, f"{what}: rel L2 {rel}"
    return float(err.max()), float(rel)


def out_to_f64(t, dtype: str) -> np.ndarray:
    return bits16_to_f64(t.cpu().contiguous().view(__import__("torch").int16).numpy().view(np.uint16), dtype)


def query_and_new(w):
    q = bits16_to_f64(w.query_bits(), w.dtype)
    kn, vn = w.new_kv_bits() if w.append else (None, None)
    return q, kn, vn


def oracle_step(w, sh, b: int, g: int, q, kn, vn, sel=None, quad=None):
    """Run the oracle step on a prepared (b, g) cache (mutates it by the append); ``quad``
    (an ``oracle.quad.QuadState``) scores pages with the quad score."""
    return step_pair(w, sh, b, g, q[b], None if kn is None else kn[b, g], None if vn is None else vn[b, g],
                     sel=sel, quad=quad)


def oracle_outputs_on(w, sh, b: int, g: int, q, pages):
    """The oracle's attention of kv head g's query heads over the given pages of a
    prepared (and already appended) cache: outputs [G, D] and lse [G]."""
    G = w.G
    idx = token_index(np.asarray(pages, dtype=np.int64), sh.L)
    out, lse = np.zeros((G, w.D)), np.zeros(G)
    for i in range(G):
        o, l, _, _ = attend(q[b, g * G + i], sh.khat[idx], sh.vhat[idx], w.sm_scale)
        out[i], lse[i] = o, l
    return out, lse


def check_unit(w, snap, scores, sel, cnt, out, lse, q, kn, vn, b: int, g: int, what: str, pages="all",
               tail: bool = True) -> bool:
    """One (sequence, kv head) unit of a GPU step against the oracle's step: the cache
    after the append (every page's bytes, or those listed in ``pages`` plus the appended
    one; summaries; the open page's key sum), the scores, the selected set and the outputs
    and lse of the G query heads.  Where the sets legitimately differ (k-th margin <= 1e-5)
    the outputs are compared with the oracle's attention over the GPU's set.  Returns
    whether the sets were equal."""
    sh = prepare(w, b, g)
    r = oracle_step(w, sh, b, g, q, kn, vn)
    P = r["P"]
    if pages == "all":
        pages = range(P)
    pages = sorted(set(int(p) for p in pages if p < P) | ({int(w.lens[b]) // 16} if w.append and P else set()))
    check_pages(snap, sh, w, b, g, pages)
    check_summary(snap, sh, b, g, P)
    if w.append or int(w.lens[b]) % 16:
        assert np.array_equal(snap["ksum"][b, g], sh.ksum), f"{what}: open-page key sum differs"
    G = w.G
    check_scores(scores[b, g], r["scores"], q[b, g * G:(g + 1) * G], sh.summary, P, tail=tail)
    got_sel = sel[b, g, :cnt[b, g]]
    same = check_selection(got_sel, r["sel"], r["scores"], w, P)
    ref_out, ref_lse = (r["out"], r["lse"]) if same else oracle_outputs_on(w, sh, b, g, q, got_sel)
    for i in range(G):
        h = g * G + i
        check_output(out[b, h], ref_out[i], f"{what} b={b} h={h}", w.dtype)
        if np.isfinite(ref_lse[i]):
            assert abs(lse[b, h] - ref_lse[i]) <= 1e-3 * max(1.0, abs(ref_lse[i])), (what, b, h)
        else:
            assert not np.isfinite(lse[b, h])
    return same


def sample_units(w, n: int, seed: int = 0):
    """n distinct (b, g) units: the first, the last, c4's longest and shortest sequences,
    then seeded draws."""
    units = {(0, 0), (w.B - 1, w.Hkv - 1)}
    if w.name == "c4":
        bl, bs = int(np.argmax(w.lens)), int(np.argmin(w.lens))
        units |= {(bl, 0), (bl, w.Hkv - 1), (bs, 0), (bs, w.Hkv - 1)}
    rng = np.random.default_rng(seed)
    while len(units) < min(n, w.B * w.Hkv):
        units.add((int(rng.integers(w.B)), int(rng.integers(w.Hkv))))
    return sorted(units)
