"""Paged cache of one (sequence, kv head): tiers, stored codes, summaries, append.

Test infrastructure only (see ``oracle/__init__.py``).

AMASS ("What is in the box") scores pages from "a tiny per-page summary"; the
summary it actually uses ("quad") is not defined on the page, so the plainest
summary is taken: the mean key of the page.  It is computed from the keys as they
arrived (before any quantisation) and stored as fp16:
``kbar[p] = fp16(S_p / n_p)`` with ``S_p`` the fp64 sum of the page's keys in token
order and ``n_p`` its number of tokens.  Appending one token to the open page adds
it to that running sum (one fp64 add), so a page built in one go and a page grown
token by token hold the same summary.

Pages hold T = 16 tokens.  Each logical page has one tier, shared by all kv heads;
16-bit pages store the cache values unchanged, the others store codes per
``oracle.quant`` in the byte order of ``oracle.layout``.
"""
from __future__ import annotations

import dataclasses

import numpy as np

from .fp import bits16_to_f64, fp16_rne_sat
from .layout import T, pack_chunk
from .quant import TIER_F16, quantise_token


@dataclasses.dataclass
class SeqHead:
    dtype: str
    D: int
    L: int
    tiers: np.ndarray          # [P_cap] tier of each logical page
    korig: np.ndarray          # [cap, D] fp64, keys as they arrived
    kbits: np.ndarray          # [cap, D] uint16 patterns (16-bit payload)
    vbits: np.ndarray
    khat: np.ndarray           # [cap, D] values read back (fp64 holding fp32/fp16/bf16)
    vhat: np.ndarray
    kcodes: np.ndarray         # [cap, D] int64 codes (b-bit pages)
    vcodes: np.ndarray
    kmeta: np.ndarray          # [cap, D/32] uint32 metadata words
    vmeta: np.ndarray
    summary: np.ndarray        # [P_cap, D] fp64 (fp16 values)
    summary_bits: np.ndarray   # [P_cap, D] uint16
    ksum: np.ndarray           # [D] fp64 running key sum of the open page
    overflow: bool = False

    @property
    def P(self) -> int:
        return (self.L + T - 1) // T


def _store(sh: SeqHead, t, tier: int, kb: np.ndarray, vb: np.ndarray):
    """Store token(s) ``t`` (an index or a slice of one page) into ``tier``."""
    k = bits16_to_f64(kb, sh.dtype)
    v = bits16_to_f64(vb, sh.dtype)
    sh.korig[t] = k
    sh.kbits[t] = kb
    sh.vbits[t] = vb
    qk = quantise_token(k, tier)
    qv = quantise_token(v, tier)
    sh.khat[t] = qk["xhat"]
    sh.vhat[t] = qv["xhat"]
    if tier != TIER_F16:
        sh.kcodes[t] = qk["codes"]
        sh.vcodes[t] = qv["codes"]
        sh.kmeta[t] = qk["meta"]
        sh.vmeta[t] = qv["meta"]
    sh.overflow |= bool(np.any(qk["overflow"]) or np.any(qv["overflow"]))


def build(kbits: np.ndarray, vbits: np.ndarray, dtype: str, tiers: np.ndarray,
          capacity_pages: int | None = None) -> SeqHead:
    """Store a prefilled context ``kbits/vbits [L, D]`` (16-bit patterns) page by page."""
    L, D = kbits.shape
    tiers = np.asarray(tiers, dtype=np.int64)
    Pc = max(capacity_pages or 0, tiers.size, (L + T - 1) // T)
    cap = Pc * T
    G = D // 32
    sh = SeqHead(dtype=dtype, D=D, L=0, tiers=np.zeros(Pc, np.int64),
                 korig=np.zeros((cap, D)), kbits=np.zeros((cap, D), np.uint16),
                 vbits=np.zeros((cap, D), np.uint16), khat=np.zeros((cap, D)),
                 vhat=np.zeros((cap, D)), kcodes=np.zeros((cap, D), np.int64),
                 vcodes=np.zeros((cap, D), np.int64), kmeta=np.zeros((cap, G), np.uint32),
                 vmeta=np.zeros((cap, G), np.uint32), summary=np.zeros((Pc, D)),
                 summary_bits=np.zeros((Pc, D), np.uint16), ksum=np.zeros(D))
    sh.tiers[: tiers.size] = tiers
    for p in range((L + T - 1) // T):
        s = slice(p * T, min(L, p * T + T))
        _store(sh, s, int(sh.tiers[p]), kbits[s], vbits[s])
    sh.L = L
    for p in range((L + T - 1) // T):
        _set_summary(sh, p)
    if L % T:
        sh.ksum = _page_sum(sh, (L - 1) // T)
    return sh


def _page_sum(sh: SeqHead, p: int) -> np.ndarray:
    """fp64 sum of the page's original keys, added one token at a time in order."""
    s = np.zeros(sh.D)
    for t in range(p * T, min(sh.L, p * T + T)):
        s = s + sh.korig[t]
    return s


def _set_summary(sh: SeqHead, p: int):
    n = min(sh.L, p * T + T) - p * T
    val, bits, ov = fp16_rne_sat(_page_sum(sh, p) / n)
    sh.summary[p] = val
    sh.summary_bits[p] = bits
    sh.overflow |= bool(np.any(ov))


def append(sh: SeqHead, pos: int, kb: np.ndarray, vb: np.ndarray):
    """Write one token at position ``pos`` (== current length) and refresh its page's summary.

    The open page's running sum restarts at a page boundary and otherwise gains the
    new key; the page summary becomes ``fp16(sum / n)``.
    """
    assert pos == sh.L, "append writes the next position"
    p, t = divmod(pos, T)
    _store(sh, pos, int(sh.tiers[p]), kb, vb)
    k = sh.korig[pos]
    sh.ksum = k.copy() if t == 0 else sh.ksum + k
    sh.L = pos + 1
    val, bits, ov = fp16_rne_sat(sh.ksum / (t + 1))
    sh.summary[p] = val
    sh.summary_bits[p] = bits
    sh.overflow |= bool(np.any(ov))


def page_bytes(sh: SeqHead, p: int, kind: str) -> np.ndarray:
    """Chunk bytes of logical page p for K ('k') or V ('v')."""
    tier = int(sh.tiers[p])
    s = p * T
    n = max(0, min(sh.L, s + T) - s)
    if tier == TIER_F16:
        pay = (sh.kbits if kind == "k" else sh.vbits)[s:s + n]
        return pack_chunk(kind, tier, sh.D, n, pay)
    pay = (sh.kcodes if kind == "k" else sh.vcodes)[s:s + n]
    meta = (sh.kmeta if kind == "k" else sh.vmeta)[s:s + n]
    return pack_chunk(kind, tier, sh.D, n, pay, meta)


def requantize(sh: SeqHead, p: int, new_tier: int):
    """Tier demotion (ARGUS "Visual Architecture": pages move down the cascade as they cool).

    Reading: the page's values as read back from its current tier (the 16-bit values, or
    ``fp32(c*scale + zero)``, or ``+-m``) are quantised again, token by token and group by
    group, with the same quantiser into ``new_tier`` (a b-bit tier).  The summary, built
    from the keys as they arrived, is unchanged.
    """
    assert new_tier != TIER_F16, "demotion goes to a b-bit tier"
    s = slice(p * T, max(p * T, min(sh.L, p * T + T)))
    for t in range(s.start, s.stop):
        qk = quantise_token(sh.khat[t].copy(), new_tier)
        qv = quantise_token(sh.vhat[t].copy(), new_tier)
        sh.khat[t], sh.vhat[t] = qk["xhat"], qv["xhat"]
        sh.kcodes[t], sh.vcodes[t] = qk["codes"], qv["codes"]
        sh.kmeta[t], sh.vmeta[t] = qk["meta"], qv["meta"]
        sh.overflow |= bool(np.any(qk["overflow"]) or np.any(qv["overflow"]))
    sh.tiers[p] = new_tier
