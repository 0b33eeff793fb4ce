"""Byte layout of one page chunk (one page, one kv head, K or V).

Test infrastructure only (see ``oracle/__init__.py``).

The pages say only that INT4 packs two codes per byte, INT2 four and 1-bit eight
(ARGUS, "Visual Architecture"; AdaptiveKV, "Architecture Overview").  The order of
the codes inside a page is this library's own choice.  It is the operand order of a
16x8x16 warp-level tensor-core multiply, so a warp reads each page with 16-byte
loads that are contiguous across lanes and needs no shuffles to form operands.

A chunk holds the T = 16 token slots of one page for one kv head, either keys (K) or
values (V), and is laid out as ``codes`` followed by ``meta``.

**Element order.**  Each element (t, d) (token slot t, channel d) is owned by one of
32 lanes ``lam`` and sits in register pair ``R = 4*kk + r`` as its ``half`` (0 = low,
1 = high), with ``kk = d // 16`` and ``c = d % 16``:

* K:  ``lam = 4*(t % 8) + (c % 8)//2``,  ``r = 2*(c // 8) + t // 8``,  ``half = c % 2``
* V:  ``lam = 4*(c % 8) + (t % 8)//2``,  ``r = 2*(t // 8) + c // 8``,  ``half = t % 2``

(K rows are tokens; V is stored transposed, rows are channels.)

**16-bit tier.**  The 16-bit value of (lam, R, half) is half ``half`` of the
little-endian uint32 word ``(kk*32 + lam)*4 + r``.

**b-bit tiers (b = 8, 4, 2, 1).**  Lane ``lam``'s pairs are packed into 32-bit words,
``16/b`` pairs per word: pair R goes to lane-word ``w = R // (16/b)`` at slot
``j = R % (16/b)``; its low code occupies bits ``[b*j, b*j + b)`` and its high code
bits ``[16 + b*j, 16 + b*j + b)``.  A lane has ``NW = D*b/64`` words; with
``PW = min(4, NW)``, lane-word w is stored at uint32 index
``((w // PW)*32 + lam)*PW + w % PW`` of the codes area.  1-bit codes are 1 for a
non-negative value.

**meta.**  INT-b: uint32 ``[T][D/32]`` = ``scale_bits | zero_bits << 16`` (fp16 bits).
1-bit: uint16 ``[T][D/32]`` magnitude (fp16 bits).  Token slots that hold no token,
and any unused bits, are zero.
"""
from __future__ import annotations

import functools

import numpy as np

from .quant import TIER_F16, TIER_F8, TIER_I1, TIER_BITS

T = 16


def codes_bytes(tier: int, D: int) -> int:
    return T * D * TIER_BITS[tier] // 8


def meta_bytes(tier: int, D: int) -> int:
    if tier == TIER_F16:
        return 0
    return T * (D // 32) * (2 if tier in (TIER_I1, TIER_F8) else 4)


def chunk_bytes(tier: int, D: int) -> int:
    return codes_bytes(tier, D) + meta_bytes(tier, D)


def element_slot(kind: str, t: np.ndarray, d: np.ndarray):
    """(lane, kk, r, half) of elements (t, d) of a K ('k') or V ('v') chunk."""
    kk = d // 16
    c = d % 16
    if kind == "k":
        lam = 4 * (t % 8) + (c % 8) // 2
        r = 2 * (c // 8) + t // 8
        half = c % 2
    else:
        lam = 4 * (c % 8) + (t % 8) // 2
        r = 2 * (t // 8) + c // 8
        half = t % 2
    return lam, kk, r, half


@functools.lru_cache(maxsize=None)
def _positions(kind: str, tier: int, D: int):
    """For every (t, d): (u32 word index into the codes area, bit offset)."""
    t, d = np.meshgrid(np.arange(T), np.arange(D), indexing="ij")
    lam, kk, r, half = element_slot(kind, t, d)
    if tier == TIER_F16:
        word = (kk * 32 + lam) * 4 + r
        return word, 16 * half
    b = TIER_BITS[tier]
    ppw = 16 // b
    R = 4 * kk + r
    w = R // ppw
    j = R % ppw
    nw = D * b // 64
    pw = min(4, nw)
    word = ((w // pw) * 32 + lam) * pw + (w % pw)
    return word, b * j + 16 * half


def pack_chunk(kind: str, tier: int, D: int, n_valid: int, payload: np.ndarray,
               meta: np.ndarray | None = None) -> np.ndarray:
    """Bytes of one chunk.

    ``payload[T', D]`` (T' = n_valid) is the 16-bit patterns (16-bit tier) or the
    integer codes (b-bit tiers) of the valid token slots; ``meta[T', D/32]`` is the
    per-group metadata word (b-bit tiers).  Returns uint8 ``[chunk_bytes]``.
    """
    nwords = codes_bytes(tier, D) // 4
    words = np.zeros(nwords, dtype=np.uint64)
    wi, bo = _positions(kind, tier, D)
    wi, bo = wi[:n_valid], bo[:n_valid]
    vals = np.asarray(payload, dtype=np.uint64)[:n_valid]
    if tier != TIER_F16:
        b = TIER_BITS[tier]
        assert np.all(vals < (1 << b))
    np.bitwise_or.at(words, wi.ravel(), (vals << bo.astype(np.uint64)).ravel())
    out = [words.astype(np.uint32).view(np.uint8)]
    if tier != TIER_F16:
        G = D // 32
        if tier in (TIER_I1, TIER_F8):
            m = np.zeros((T, G), dtype=np.uint16)
            m[:n_valid] = np.asarray(meta, dtype=np.uint16)[:n_valid]
        else:
            m = np.zeros((T, G), dtype=np.uint32)
            m[:n_valid] = np.asarray(meta, dtype=np.uint32)[:n_valid]
        out.append(m.view(np.uint8).ravel())
    return np.concatenate(out)


def unpack_chunk(kind: str, tier: int, D: int, data: np.ndarray):
    """Inverse of ``pack_chunk`` for all T slots: ``(payload[T, D], meta[T, D/32] | None)``."""
    data = np.asarray(data, dtype=np.uint8)
    cb = codes_bytes(tier, D)
    words = data[:cb].view(np.uint32).astype(np.uint64)
    wi, bo = _positions(kind, tier, D)
    mask = 0xFFFF if tier == TIER_F16 else (1 << TIER_BITS[tier]) - 1
    payload = (words[wi] >> bo.astype(np.uint64)) & np.uint64(mask)
    meta = None
    if tier != TIER_F16:
        G = D // 32
        dt = np.uint16 if tier in (TIER_I1, TIER_F8) else np.uint32
        meta = data[cb:].view(dt).reshape(T, G)
    return payload.astype(np.int64), meta
