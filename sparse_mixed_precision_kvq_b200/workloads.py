"""Seeded synthetic inputs for sparse mixed-precision paged decode attention.

This module only draws numbers: keys, values, queries, context lengths, page tier
assignments and physical slot maps.  It holds none of the method's arithmetic
(no quantisation, summary, scoring, selection or attention), so that the CUDA
path and the CPU oracle can both be fed from it without sharing any computation.

Every random stream is a numpy PCG64 generator keyed by
``SeedSequence([seed, stream_tag, *indices])``, so any (sequence, kv head) slice can
be regenerated on its own without drawing the rest of the cache.

Workload recipes (page size T = 16 everywhere):

* ``c0``  tiny: 1 sequence, 8 q / 2 kv heads, D 64, 1024 tokens, fp16, all pages
  16-bit, 4 planted pages, top-8 + page 0 + last page.
* ``c1``  Llama-3-8B-shaped layer: batch 8, 32 q / 8 kv heads, D 128, 32768 tokens,
  bf16, all pages 16-bit, 4 outlier channels per kv head scaled x8, 1% planted pages,
  5% selection + sink page + 4 recent pages, 1 appended token per sequence.
* ``c2``  c1's shape and laws with tiers 16-bit/int8/int4/int2 = 10/20/30/40 % by a
  seeded rank, 10% selection, 1 appended token per sequence.
* ``c3``  batch 1, 32 q / 8 kv heads, D 128, 131072 tokens, bf16, physical slots
  randomly permuted, int4 cold pages, 16-bit hot pages (a seeded 5% hot set, planted
  so that the selector picks it, plus the sink and 16 most recent pages).
* ``c4``  ragged Qwen2.5-3B-shaped layer: batch 64, 16 q / 2 kv heads, D 128, bf16,
  context lengths log-uniform in [2048, 65536], tiers 16-bit/int4/int2/1-bit =
  10/30/40/20 %, 8% selection + sink + 4 recent, outlier key channels.

Planted pages hold keys ``2.4 * qhat + eps`` where ``qhat`` is the unit vector of the
first query head of the kv head's group and ``eps`` follows the workload's key law.

Overrides used by the tests and the benchmark: ``tier_fracs`` (any mix of the six tiers,
fp8 included, assigned by seeded rank; ``{T: 1.0}`` puts every prefilled page at tier T),
reduced batch / lengths (``small``), and ``quad_basis`` (the quad score's per-kv-head
basis: unit vectors along the key law's largest-variance channels, or a seeded random
orthonormal set).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import numpy as np

PAGE = 16
TIER_F16, TIER_I8, TIER_I4, TIER_I2, TIER_I1, TIER_F8 = 0, 1, 2, 3, 4, 5
N_TIERS = 6

# stream tags (part of the seed key of each random stream)
_S_KEY, _S_VAL, _S_Q, _S_KNEW, _S_VNEW, _S_OUTL, _S_PLANT, _S_TIER, _S_SLOT, _S_LEN, _S_QUAD = range(11)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round-half-even) and return the 16-bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def f32_to_f16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to IEEE fp16 (round-half-even) and return the 16-bit patterns."""
    return np.ascontiguousarray(x, dtype=np.float32).astype(np.float16).view(np.uint16)


def bits_to_f32(bits: np.ndarray, dtype: str) -> np.ndarray:
    """Widen 16-bit patterns of ``dtype`` ('f16' or 'bf16') to float32 (exact)."""
    bits = np.asarray(bits, dtype=np.uint16)
    if dtype == "f16":
        return bits.view(np.float16).astype(np.float32)
    return (bits.astype(np.uint32) << 16).view(np.float32)


def _rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, *key])))


@dataclasses.dataclass
class Workload:
    """One decode step's synthetic inputs (metadata + lazily drawn tensors)."""

    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    dtype: str                    # 'f16' | 'bf16' (cache, query and output dtype)
    lens: np.ndarray              # [B] int64, tokens in the cache before the step's append
    append: bool                  # whether the step appends one token per sequence
    k_abs: int                    # >= 0: absolute top-k; -1: use k_frac_bp
    k_frac_bp: int                # top-k fraction in basis points (used when k_abs < 0)
    n_sink: int                   # forced leading pages
    n_recent: int                 # forced trailing pages
    seed: int
    outlier_channels: int = 0     # key channels per kv head scaled by outlier_scale
    outlier_scale: float = 8.0
    plant_frac: float = 0.0       # fraction of pages per sequence planted (floor)
    plant_count: int = 0          # absolute planted page count (overrides plant_frac)
    plant_lo: int = 1             # planted pages are drawn from [plant_lo, P - plant_hi_gap)
    plant_hi_gap: int = 1
    tier_fracs: Optional[Dict[int, float]] = None   # tier -> fraction, by seeded rank
    hot_f16_planted: bool = False  # c3: 16-bit = planted set + sink + recent, rest int4
    hot_recent: int = 0
    permute_slots: bool = False
    T: int = PAGE

    # ---------------------------------------------------------------- shapes
    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    def final_lens(self) -> np.ndarray:
        """Context lengths after the step's append (the lengths attention runs over)."""
        return self.lens + (1 if self.append else 0)

    def pages_before(self, b: int) -> int:
        return (int(self.lens[b]) + self.T - 1) // self.T

    def pages_after(self, b: int) -> int:
        return (int(self.final_lens()[b]) + self.T - 1) // self.T

    @property
    def max_pages(self) -> int:
        return int(max(self.pages_after(b) for b in range(self.B))) if self.B else 0

    def kmax(self) -> int:
        """Host-side upper bound on the number of pages selected per (sequence, kv head)."""
        P = self.max_pages
        k = self.k_abs if self.k_abs >= 0 else (P * self.k_frac_bp + 9999) // 10000
        return max(1, min(P, k + self.n_sink + self.n_recent))

    # ---------------------------------------------------------------- draws
    def _normal(self, tag: int, *idx: int, n: int) -> np.ndarray:
        return _rng(self.seed, tag, *idx).standard_normal((n, self.D), dtype=np.float32)

    def _to_bits(self, x: np.ndarray) -> np.ndarray:
        return f32_to_bf16_bits(x) if self.dtype == "bf16" else f32_to_f16_bits(x)

    def outlier_idx(self, g: int) -> np.ndarray:
        if self.outlier_channels <= 0:
            return np.zeros(0, dtype=np.int64)
        r = _rng(self.seed, _S_OUTL, g)
        return np.sort(r.choice(self.D, size=self.outlier_channels, replace=False))

    def quad_basis(self, g: int, rank: int, kind: str = "law") -> np.ndarray:
        """Basis rows of kv head g for the quad page score, fp32 ``[rank, D]``.

        ``law``: unit vectors along the channels of largest key variance under this
        workload's key law (its outlier channels, then the others in index order) -- the
        eigenvectors of the law's diagonal covariance.  ``random``: a seeded random
        orthonormal set (QR of a Gaussian matrix)."""
        if kind == "random":
            a = _rng(self.seed, _S_QUAD, g).standard_normal((self.D, self.D))
            qm, _ = np.linalg.qr(a)
            return np.ascontiguousarray(qm[:, :rank].T).astype(np.float32)
        first = [int(c) for c in self.outlier_idx(g)]
        chans = (first + [c for c in range(self.D) if c not in first])[:rank]
        u = np.zeros((rank, self.D), dtype=np.float32)
        u[np.arange(rank), chans] = 1.0
        return u

    def query_bits(self) -> np.ndarray:
        """q [B, Hq, D] as 16-bit patterns of the workload dtype."""
        q = _rng(self.seed, _S_Q).standard_normal((self.B, self.Hq, self.D), dtype=np.float32)
        return self._to_bits(q)

    def planted_pages(self, b: int) -> np.ndarray:
        """Logical pages of sequence b whose keys are planted (same for every kv head)."""
        P = self.pages_before(b)
        if self.plant_count > 0:
            n = self.plant_count
        else:
            n = int(math.floor(self.plant_frac * P))
        lo, hi = self.plant_lo, P - self.plant_hi_gap
        if n <= 0 or hi <= lo:
            return np.zeros(0, dtype=np.int64)
        n = min(n, hi - lo)
        r = _rng(self.seed, _S_PLANT, b)
        return np.sort(lo + r.choice(hi - lo, size=n, replace=False))

    def _key_law(self, x: np.ndarray, g: int) -> np.ndarray:
        idx = self.outlier_idx(g)
        if idx.size:
            x[:, idx] *= np.float32(self.outlier_scale)
        return x

    def keys_bits(self, b: int, g: int) -> np.ndarray:
        """Prefilled keys of (sequence b, kv head g): [lens[b], D] 16-bit patterns."""
        L = int(self.lens[b])
        x = self._key_law(self._normal(_S_KEY, b, g, n=L), g)
        pp = self.planted_pages(b)
        if pp.size:
            q = bits_to_f32(self.query_bits()[b, g * self.G], self.dtype).astype(np.float64)
            qhat = (q / np.sqrt(np.sum(q * q))).astype(np.float32)
            for p in pp:
                s, e = p * self.T, min(L, p * self.T + self.T)
                x[s:e] += np.float32(2.4) * qhat
        return self._to_bits(x)

    def values_bits(self, b: int, g: int) -> np.ndarray:
        """Prefilled values of (sequence b, kv head g): [lens[b], D] 16-bit patterns."""
        return self._to_bits(self._normal(_S_VAL, b, g, n=int(self.lens[b])))

    def new_kv_bits(self):
        """The appended token's (k_new, v_new), each [B, Hkv, D] 16-bit patterns."""
        k = np.empty((self.B, self.Hkv, self.D), dtype=np.float32)
        for g in range(self.Hkv):
            k[:, g, :] = self._key_law(
                _rng(self.seed, _S_KNEW, g).standard_normal((self.B, self.D), dtype=np.float32), g)
        v = _rng(self.seed, _S_VNEW).standard_normal((self.B, self.Hkv, self.D), dtype=np.float32)
        return self._to_bits(k), self._to_bits(v)

    # ---------------------------------------------------------------- tiers
    def tiers(self, b: int) -> np.ndarray:
        """Tier of every logical page of sequence b after the append: uint8 [pages_after(b)]."""
        P0, P1 = self.pages_before(b), self.pages_after(b)
        t = np.zeros(P1, dtype=np.uint8)
        if self.hot_f16_planted:
            t[:] = TIER_I4
            t[self.planted_pages(b)] = TIER_F16
            t[: min(self.n_sink, P1)] = TIER_F16
            t[max(0, P1 - self.hot_recent):] = TIER_F16
        elif self.tier_fracs:
            perm = _rng(self.seed, _S_TIER, b).permutation(P0)
            order = sorted(self.tier_fracs.items())
            cum, start = 0.0, 0
            for tier, frac in order:
                cum += frac
                end = P0 if tier == order[-1][0] else int(math.floor(cum * P0 + 1e-9))
                t[perm[start:end]] = tier
                start = end
        if P1 > P0:                       # a page opened by the append starts 16-bit
            t[P0:] = TIER_F16
        return t

    def slot_map(self):
        """Physical placement: (block_table int64 [B, max_pages] of (tier, slot)), pool slot counts.

        Returns ``(tier_tbl, slot_tbl, pool_slots)`` where unused entries are -1.
        """
        MP = self.max_pages
        tier_tbl = np.full((self.B, MP), -1, dtype=np.int64)
        slot_tbl = np.full((self.B, MP), -1, dtype=np.int64)
        counts = [0] * N_TIERS
        for b in range(self.B):
            tb = self.tiers(b)
            tier_tbl[b, : tb.size] = tb
            for p, tr in enumerate(tb):
                slot_tbl[b, p] = counts[tr]
                counts[tr] += 1
        if self.permute_slots:
            for tr in range(N_TIERS):
                if counts[tr] == 0:
                    continue
                perm = _rng(self.seed, _S_SLOT, tr).permutation(counts[tr])
                m = tier_tbl == tr
                slot_tbl[m] = perm[slot_tbl[m]]
        return tier_tbl, slot_tbl, counts


def _loguniform_lens(seed: int, B: int, lo: int, hi: int) -> np.ndarray:
    u = _rng(seed, _S_LEN).uniform(math.log(lo), math.log(hi), size=B)
    return np.floor(np.exp(u)).astype(np.int64)


def make(name: str, **over) -> Workload:
    """Build a named workload; keyword overrides shrink it for tests (B, lens, ...)."""
    name = name.lower()
    base_seed = 0xC0FFEE
    if name == "c0":
        w = dict(B=1, Hq=8, Hkv=2, D=64, dtype="f16", lens=np.array([1024]), append=False,
                 k_abs=8, k_frac_bp=0, n_sink=1, n_recent=1, seed=base_seed + 0,
                 plant_count=4, plant_lo=1, plant_hi_gap=1)
    elif name == "c1":
        w = dict(B=8, Hq=32, Hkv=8, D=128, dtype="bf16", lens=np.full(8, 32768), append=True,
                 k_abs=-1, k_frac_bp=500, n_sink=1, n_recent=4, seed=base_seed + 1,
                 outlier_channels=4, plant_frac=0.01, plant_lo=1, plant_hi_gap=4)
    elif name == "c2":
        w = dict(B=8, Hq=32, Hkv=8, D=128, dtype="bf16", lens=np.full(8, 32768), append=True,
                 k_abs=-1, k_frac_bp=1000, n_sink=1, n_recent=4, seed=base_seed + 2,
                 outlier_channels=4, plant_frac=0.01, plant_lo=1, plant_hi_gap=4,
                 tier_fracs={TIER_F16: 0.1, TIER_I8: 0.2, TIER_I4: 0.3, TIER_I2: 0.4})
    elif name == "c3":
        w = dict(B=1, Hq=32, Hkv=8, D=128, dtype="bf16", lens=np.array([131072]), append=True,
                 k_abs=-1, k_frac_bp=500, n_sink=1, n_recent=16, seed=base_seed + 3,
                 plant_count=410, plant_lo=1, plant_hi_gap=16, hot_f16_planted=True,
                 hot_recent=16, permute_slots=True)
    elif name == "c4":
        w = dict(B=64, Hq=16, Hkv=2, D=128, dtype="bf16", lens=None, append=True,
                 k_abs=-1, k_frac_bp=800, n_sink=1, n_recent=4, seed=base_seed + 4,
                 outlier_channels=4,
                 tier_fracs={TIER_F16: 0.1, TIER_I4: 0.3, TIER_I2: 0.4, TIER_I1: 0.2})
    else:
        raise ValueError(f"unknown workload {name!r}")
    lens_range = over.pop("lens_range", None)
    w.update(over)
    if name == "c4" and w.get("lens") is None:
        lo, hi = lens_range or (2048, 65536)
        w["lens"] = _loguniform_lens(w["seed"], w["B"], lo, hi)
    elif lens_range is not None:
        w["lens"] = _loguniform_lens(w["seed"], w["B"], *lens_range)
    w["lens"] = np.asarray(w["lens"], dtype=np.int64)
    if w["lens"].size != w["B"]:
        w["lens"] = np.resize(w["lens"], w["B"]).astype(np.int64)
    # c3 plants the same number of pages as its selection budget takes
    if name == "c3" and "plant_count" not in over:
        P = int((w["lens"][0] + PAGE) // PAGE) if w["append"] else int((w["lens"][0] + PAGE - 1) // PAGE)
        w["plant_count"] = (P * w["k_frac_bp"] + 9999) // 10000
    return Workload(name=name, **w)


# Reduced shapes used by the parity tests: same per-element laws, tiers and selection
# rules as the full workloads, sized so the CPU oracle finishes in seconds while still
# spanning many pages, several split-K chunks and ragged tails.
SMALL = {
    "c0": dict(),
    "c1": dict(B=2, lens=np.array([2048, 2048])),
    "c2": dict(B=2, lens=np.array([2048, 1000])),
    "c3": dict(lens=np.array([8192])),
    "c4": dict(B=6, lens_range=(40, 3000)),
}


def small(name: str, **over) -> Workload:
    kw = dict(SMALL[name.lower()])
    kw.update(over)
    return make(name, **kw)
