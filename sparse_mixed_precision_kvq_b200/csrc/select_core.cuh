// Per-(sequence, kv head) page selection, block-wide, shared by kvq_select_topk and the
// fused decode step.
//
// AMASS "Quickstart" (budget: a fixed fraction of the pages is attended, here rounded
// up per sequence: k = ceil(P * bp / 10000)); ARGUS "Quickstart" (sink tokens kept) and
// "The One-Minute Explanation" (recent tokens stay hot): the first n_sink and last
// n_recent pages are always attended, in addition to the k best other pages.  Ranking:
// score descending, lower page index first among equal scores, NaN lowest.
//
// Scores are mapped to order-preserving 32-bit keys in shared memory.  The chosen
// candidates are found exactly in two steps.  (1) A 256-bin histogram of the candidates'
// scores, binned linearly between their minimum and maximum (NaN in a bin of its own,
// below all others), locates the bin T that holds the k-th largest and how many of T's
// pages are chosen; the binning is monotone in the score, so every page of a higher bin is
// chosen and none of a lower one.  (2) The pages of bin T -- a few, for any spread-out
// score distribution -- are ranked against each other by (key descending, page
// ascending).  The choice is a bitmap of pages, built 32 pages per warp ballot; one
// block scan over its words then emits the chosen pages in ascending order.  When bin T
// holds more than kSelCand pages (heavy ties, or an infinite score range), an MSB-first
// radix select over the keys (4 passes of 8 bits) finds the threshold key instead.
// Ties are resolved on the keys; the binning decides nothing by itself.
#pragma once

#include <math.h>

#include "kvq_internal.cuh"

namespace kvq {

// Order-preserving key of a score (larger score -> larger key); NaN -> 0 and *nan set.
__device__ inline uint32_t order_key(float f, bool& nan) {
  if (isnan(f)) {
    nan = true;
    return 0u;
  }
  if (f == 0.0f) f = 0.0f;  // -0 and +0 rank equal
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The split of P pages: forced pages [0, ns) and [rs, P), nC candidates, kk of them chosen.
struct SelectSplit {
  int ns, rs, nC, kk;
  __host__ __device__ int count(int P) const { return (P - nC) + kk; }
};

__host__ __device__ inline SelectSplit select_split(int P, const kvq_select_params& prm) {
  SelectSplit s;
  s.ns = min(max(prm.n_sink, 0), P);
  s.rs = max(P - max(prm.n_recent, 0), 0);
  const int nF = s.ns + (P - s.rs) - max(0, s.ns - s.rs);
  s.nC = P - nF;
  const long long kb = prm.k_abs >= 0 ? (long long)prm.k_abs : ((long long)P * prm.k_frac_bp + 9999) / 10000;
  const long long kb0 = kb < 0 ? 0 : kb;
  s.kk = static_cast<int>(kb0 < s.nC ? kb0 : s.nC);
  return s;
}

constexpr int kSelBins = 256;      // value-linear histogram bins (+1 for NaN)
constexpr int kSelCand = 1024;     // most pages of the threshold bin ranked directly
constexpr int kSelCandOff = 288;   // scratch: [0, 257) histogram, then candidates, then the bitmap
constexpr int kSelBitmapOff = kSelCandOff + 2 * kSelCand;
constexpr int kSelScratchWords = 4096;  // scratch words: bitmap of up to (4096 - 2336) * 32 pages
constexpr int kSelMaxPages = (kSelScratchWords - kSelBitmapOff) * 32;

struct SelShared {
  int hist[256];  // radix fallback
  int scan[33];
  float wmin[32], wmax[32];
  double dsum[33];
  uint32_t prefix;
  int rem;
  int ncand;
  // coverage selection
  unsigned long long ckmin, ckmax, cabove;
  int cbin, ccount;
};

// Exclusive prefix sum of one int per thread over NT threads; *total receives the sum.
// `bar` is the block barrier.
template <int NT, typename Bar>
__device__ inline int sel_exclusive_scan(int v, SelShared& sh, int* total, int tid, Bar& bar) {
  constexpr int NW = NT / 32;
  const int lane = tid & 31, warp = tid >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh.scan[warp] = x;
  bar();
  if (warp == 0) {
    int w = lane < NW ? sh.scan[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < NW) sh.scan[lane] = w;
  }
  bar();
  const int before = (warp ? sh.scan[warp - 1] : 0) + x - v;
  *total = sh.scan[NW - 1];
  bar();
  return before;
}

// Score of an order key (inverse of order_key; key 0 stands for NaN).
__device__ inline float key_score(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Write the pages of a bitmap (nwords words) in ascending order to out[0 .. min(n, kmax)),
// min(n, kmax) to *cnt_out (thread 0); flags KVQ_DERR_KMAX if n > kmax.
template <int NT, typename Bar>
__device__ inline void emit_chosen(const uint32_t* chosen, int nwords, int32_t* out, int32_t* cnt_out, int kmax,
                                   uint32_t* err, SelShared& sh, int tid, Bar& bar) {
  const int WPT = (nwords + NT - 1) / NT;  // contiguous words per thread
  const int w_lo = min(nwords, tid * WPT), w_hi = min(nwords, w_lo + WPT);
  int nsel = 0;
  for (int wd = w_lo; wd < w_hi; ++wd) nsel += __popc(chosen[wd]);
  int total;
  int off = sel_exclusive_scan<NT>(nsel, sh, &total, tid, bar);
  for (int wd = w_lo; wd < w_hi; ++wd) {
    unsigned m = chosen[wd];
    while (m) {
      const int b = __ffs(m) - 1;
      m &= m - 1u;
      if (off < kmax) out[off] = 32 * wd + b;
      ++off;
    }
  }
  if (tid == 0) {
    *cnt_out = min(total, kmax);
    if (total > kmax) set_err(err, KVQ_DERR_KMAX);
  }
}

// Value bin of a candidate key between the candidates' minimum lo and 256 / range sc
// (sc == 0: a single bin); NaN (key 0) in bin 256, below all others.
__device__ inline int sel_bin(uint32_t k, float lo, float sc) {
  if (k == 0u) return 256;  // NaN
  const float v = (key_score(k) - lo) * sc;
  return v >= 255.f ? 255 : (v > 0.f ? static_cast<int>(v) : 0);
}

// 256 / range of the candidates' scores [lo, hi], or 0 (one bin) when the range is empty,
// zero or not finite.
__device__ inline float sel_scale(float lo, float hi) {
  const float range = hi - lo;
  float scale = (range > 0.f && range <= 3.0e38f) ? 256.f / range : 0.f;
  if (!(scale <= 3.0e38f)) scale = 0.f;
  return scale;
}

// Warp 0 (lane = its lane): the bin T that holds the kk-th largest candidate (bins in rank
// order 255 .. 0, then the NaN bin 256) and how many of T's pages are chosen, into
// sh.prefix and sh.rem.
__device__ inline void sel_find_bin(const int* hist, int kk, SelShared& sh, int lane) {
  int h[8], tot = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    h[i] = hist[255 - (lane * 8 + i)];
    tot += h[i];
  }
  int x = tot;  // inclusive prefix over lanes
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  int cum = x - tot;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (cum < kk && kk <= cum + h[i]) {
      sh.prefix = static_cast<uint32_t>(255 - (lane * 8 + i));
      sh.rem = kk - cum;
    }
    cum += h[i];
  }
  if (lane == 31 && cum < kk) {  // the NaN bin
    sh.prefix = 256u;
    sh.rem = kk - cum;
  }
}

// Warp 0: the radix digit (bits shift .. shift + 7) of the r-th largest key among those
// matching `prefix` above it, from the digit histogram; new prefix and rank into
// sh.prefix, sh.rem.
__device__ inline void sel_find_digit(const int* hist, uint32_t prefix, int shift, int r, SelShared& sh, int lane) {
  int h8[8], tot = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    h8[i] = hist[lane * 8 + i];
    tot += h8[i];
  }
  int suf = tot;  // sum over lanes >= lane
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_down_sync(0xffffffffu, suf, o);
    if (lane + o < 32) suf += y;
  }
  int cum = suf - tot;  // keys in bins above this lane's bins
#pragma unroll
  for (int i = 7; i >= 0; --i) {
    const int nxt = cum + h8[i];
    if (cum < r && r <= nxt) {
      sh.prefix = prefix | (static_cast<uint32_t>(lane * 8 + i) << shift);
      sh.rem = r - cum;
    }
    cum = nxt;
  }
}

// Select among the P keys in shared memory (written, and a barrier passed, by the
// caller); writes the chosen pages in ascending order to out[0 .. min(n, kmax)) and
// min(n, kmax) to *cnt_out (thread 0).  Flags KVQ_DERR_KMAX if n > kmax.  `scratch` is
// kSelScratchWords words of shared memory; P <= kSelMaxPages.
// PRE: the caller has already, before that barrier, put each warp's range of its
// candidates' scores (NaN left out, -0 as +0; +inf/-inf when it has none) in
// sh.wmin/sh.wmax, cleared scratch[0 .. 257) and set sh.ncand = 0 -- the first pass and
// its barrier are then skipped.
template <int NT, bool PRE = false, typename Bar>
__device__ inline void select_pages(const uint32_t* keys, int P, const kvq_select_params& prm, int32_t* out,
                                    int32_t* cnt_out, int kmax, uint32_t* err, uint32_t* scratch, SelShared& sh,
                                    int tid, Bar& bar) {
  constexpr int NW = NT / 32;
  constexpr int U = 4;  // words per warp in flight in the page passes
  const int lane = tid & 31, warp = tid >> 5;
  const SelectSplit sp = select_split(P, prm);
  const int ns = sp.ns, rs = sp.rs, nC = sp.nC, kk = sp.kk;
  const int nwords = (P + 31) / 32;
  auto is_cand = [&](int p) { return p >= ns && p < rs; };
  // f(page, valid) over all pages, page = 32 * word + lane, U words per warp at a time
  auto pages = [&](auto&& f) {
    for (int w0 = warp; w0 < nwords; w0 += U * NW) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int wd = w0 + u * NW;
        const int p = 32 * wd + lane;
        f(wd, p, wd < nwords && p < P);
      }
    }
  };

  // mode 0: no candidate chosen, 1: every candidate, 2: value bins + ranked bin T,
  // 3: threshold key from the radix select (thr, need)
  int mode = (kk == 0) ? 0 : (kk == nC ? 1 : 2);
  int* hist = reinterpret_cast<int*>(scratch);            // [257]: bin 256 = NaN
  uint32_t* cand = scratch + kSelCandOff;                 // [kSelCand][2] (key, page)
  uint32_t* chosen = scratch + kSelBitmapOff;             // [nwords] bitmap of chosen pages
  float smin = 0.f, scale = 0.f;
  uint32_t thr = 0;
  int need = 0;
  auto bin_of = [](uint32_t k, float lo, float sc) -> int { return sel_bin(k, lo, sc); };
  if (mode == 2) {
    // 1) candidates' score range; clear the histogram
    float lo = INFINITY, hi = -INFINITY;
    if constexpr (!PRE) {
      pages([&](int, int p, bool valid) {
        const uint32_t k = valid ? keys[p] : 0u;
        if (valid && is_cand(p) && k != 0u) {
          const float f = key_score(k);
          lo = fminf(lo, f);
          hi = fmaxf(hi, f);
        }
      });
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
      }
      if (lane == 0) {
        sh.wmin[warp] = lo;
        sh.wmax[warp] = hi;
      }
      for (int i = tid; i < 257; i += NT) hist[i] = 0;
      if (tid == 0) sh.ncand = 0;
      bar();
    }
    lo = INFINITY;
    hi = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      lo = fminf(lo, sh.wmin[w]);
      hi = fmaxf(hi, sh.wmax[w]);
    }
    smin = lo;
    scale = sel_scale(lo, hi);  // 0: one bin (then the radix select)
    // 2) histogram (shared atomics; the bins of a warp's pages are mostly distinct)
    pages([&](int, int p, bool valid) {
      if (valid && is_cand(p)) atomicAdd(&hist[bin_of(keys[p], smin, scale)], 1);
    });
    bar();
    // 3) warp 0: bin T holding the kk-th largest (bins in rank order: 255 .. 0, then NaN)
    if (warp == 0) sel_find_bin(hist, kk, sh, lane);
    bar();
    const int T = static_cast<int>(sh.prefix);
    const int rem = sh.rem;
    // 4) the bitmap of pages chosen outright (forced, or a bin above T), and the pages of
    //    bin T as (key, page) pairs
    pages([&](int wd, int p, bool valid) {
      const uint32_t k = valid ? keys[p] : 0u;
      const bool c = valid && is_cand(p);
      const int bk = c ? bin_of(k, smin, scale) : -1;
      const bool take = valid && (!c || (bk != T && bk != 256 && (T == 256 || bk > T)));
      const bool hit = c && bk == T;
      const unsigned tm = __ballot_sync(0xffffffffu, take);
      const unsigned hm = __ballot_sync(0xffffffffu, hit);
      if (lane == 0 && wd < nwords) chosen[wd] = tm;
      if (hm) {
        int first = 0;
        if (lane == 0) first = atomicAdd(&sh.ncand, __popc(hm));
        first = __shfl_sync(0xffffffffu, first, 0);
        if (hit) {
          const int i = first + __popc(hm & ((1u << lane) - 1u));
          if (i < kSelCand) {
            cand[2 * i] = k;
            cand[2 * i + 1] = static_cast<uint32_t>(p);
          }
        }
      }
    });
    bar();
    const int nc = sh.ncand;
    if (nc <= kSelCand) {
      // 5) rank the pages of bin T (key descending, page ascending); the first rem are chosen
      for (int i = tid; i < nc; i += NT) {
        const uint32_t ki = cand[2 * i], pi = cand[2 * i + 1];
        int rank = 0;
#pragma unroll 4
        for (int j = 0; j < nc; ++j) {
          const uint32_t kj = cand[2 * j], pj = cand[2 * j + 1];
          rank += kj > ki || (kj == ki && pj < pi);
        }
        if (rank < rem) atomicOr(&chosen[pi >> 5], 1u << (pi & 31));
      }
      bar();
    } else {
      // heavy ties: MSB-first radix select over all candidate keys
      mode = 3;
      uint32_t prefix = 0;
      int r = kk;
      for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += NT) sh.hist[i] = 0;
        bar();
        const uint32_t hmask = (shift == 24) ? 0u : (0xFFFFFFFFu << (shift + 8));
        pages([&](int, int p, bool valid) {
          if (valid && is_cand(p)) {
            const uint32_t k = keys[p];
            if ((k & hmask) == (prefix & hmask)) atomicAdd(&sh.hist[(k >> shift) & 255u], 1);
          }
        });
        bar();
        if (warp == 0) sel_find_digit(sh.hist, prefix, shift, r, sh, lane);
        bar();
        prefix = sh.prefix;
        r = sh.rem;
        bar();
      }
      thr = prefix;
      need = r;
    }
  }
  if (mode != 2) {
    // bitmap of the chosen pages: forced ones, plus every candidate (mode 1), none (mode
    // 0), or those above the threshold key (mode 3; the keys equal to it come next)
    pages([&](int wd, int p, bool valid) {
      const bool c = valid && is_cand(p);
      const bool take = valid && (!c || mode == 1 || (mode == 3 && keys[p] > thr));
      const unsigned tm = __ballot_sync(0xffffffffu, take);
      if (lane == 0 && wd < nwords) chosen[wd] = tm;
    });
    bar();
  }
  // contiguous words per thread
  const int WPT = (nwords + NT - 1) / NT;
  const int w_lo = min(nwords, tid * WPT), w_hi = min(nwords, w_lo + WPT);
  if (mode == 3) {  // the keys equal to the threshold are taken in page order, `need` of them
    auto eq_mask = [&](int wd) {
      unsigned m = 0u;
      for (int b = 0; b < 32; ++b) {
        const int p = 32 * wd + b;
        if (p < P && is_cand(p) && keys[p] == thr) m |= 1u << b;
      }
      return m;
    };
    int eq = 0;
    for (int wd = w_lo; wd < w_hi; ++wd) eq += __popc(eq_mask(wd));
    int tot_eq;
    int e = sel_exclusive_scan<NT>(eq, sh, &tot_eq, tid, bar);
    for (int wd = w_lo; wd < w_hi && e < need; ++wd) {
      unsigned m = eq_mask(wd), add = 0u;
      while (m && e < need) {
        const unsigned bit = m & (0u - m);
        add |= bit;
        m ^= bit;
        ++e;
      }
      chosen[wd] |= add;
    }
    bar();
  }
  emit_chosen<NT>(chosen, nwords, out, cnt_out, kmax, err, sh, tid, bar);
}

// ----------------------------------------------------------------------------- coverage
// AMASS "Quickstart" (coverage = 0.95, the nucleus variant of the selection).  A page's
// attention mass is estimated from its score as n_p * exp(sm_scale * (s_p - s_max)) (fp64;
// n_p its valid tokens; NaN -> 0); the forced pages count as covered, and candidates are
// added by mass (larger first, lower page first on ties) until the covered mass reaches
// coverage * the total.
//
// The chosen set is found without sorting, by an MSB-first radix search over the masses'
// fp64 bit patterns (non-negative doubles order like their bits).  Each pass histograms
// the candidates still undecided by the next (up to) 8 bits of their key, with a count and
// a mass sum per bin, and one warp finds the bin in which the running mass, taken from the
// heaviest bin down, reaches the target: heavier bins are chosen whole, lighter ones not,
// and the search continues inside that bin until it holds one page or one exact mass (then
// its lowest pages are taken, as many as reach the target).  The bin sums are fixed-point
// integers (units of 2^-46, rounded down), kept as three 17-bit parts in 32-bit counters (a
// mass is at most 16 = 2^50 units, so 8192 candidates sum below 2^30 in each part); they do
// not depend on the order of the additions, and the selection is deterministic.  A warp
// whose 32 candidates fall in at most 4 bins first merges the lanes of each bin (match +
// warp reductions), so a bin that takes most candidates sees one shared atomic per warp,
// not one per page; a warp spread over more bins adds lane by lane (warp reductions whose
// lanes name many different groups ran several times slower).  Rounding 8192 masses down
// loses under 2^-33 of a total of at least 1 (the page of the largest score has mass >= 1),
// so the cut moves only where the covered mass is that close to the target.  Candidates
// of zero mass are never taken: with coverage <= 1 the positive masses reach
// the target in exact arithmetic, so when the rounded sums fall short of it (coverage 1)
// every candidate of positive mass is taken, and no other.

constexpr int kCovMaxCand = 8192;  // candidates of one sequence (their mass keys sit in shared memory)
constexpr int kCovFixBits = 46;    // fixed-point fraction bits of the bin sums
constexpr int kCovEqOff = 1024;    // scratch: [0, 768) bin sums (3 parts), [768, 1024) counts, then the cut's pages
constexpr int kCovMaxPages = (kSelBitmapOff - kCovEqOff) * 32;  // pages whose cut bitmap fits before the bitmap

// Sum of one double per thread (fixed tree: the same order in every call).
template <int NT, typename Bar>
__device__ inline double sel_block_sum(double v, SelShared& sh, int tid, Bar& bar) {
  constexpr int NW = NT / 32;
  const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) sh.dsum[warp] = v;
  bar();
  double t = 0.0;
#pragma unroll
  for (int w = 0; w < NW; ++w) t += sh.dsum[w];
  bar();
  return t;
}

// Fixed-point mass (units of 2^-kCovFixBits, rounded down) of a mass key.
static_assert(kCovFixBits == 46, "cov_fixed and the target scale by 2^46");
__device__ inline unsigned long long cov_fixed(unsigned long long key) {
  return __double2ull_rz(__longlong_as_double(static_cast<long long>(key)) * 0x1p46);
}

// Warp 0: the bin where the running mass from the top bin down first reaches need_q (the
// mass above the bins is `above`), into sh.cbin (-1: the bins never reach it), sh.cabove
// (the mass above that bin) and sh.ccount (its pages).  bs: the bins' three sum parts.
__device__ inline void cov_find_bin(const uint32_t* bs, const int* bcnt, unsigned long long above,
                                    unsigned long long need_q, SelShared& sh, int lane) {
  unsigned long long s8[8], own = 0ull;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int b = 8 * lane + i;
    s8[i] = static_cast<unsigned long long>(bs[b]) + (static_cast<unsigned long long>(bs[256 + b]) << 17) +
            (static_cast<unsigned long long>(bs[512 + b]) << 34);
    own += s8[i];
  }
  unsigned long long suf = own;  // mass of this lane's bins and every higher lane's
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_down_sync(0xffffffffu, suf, o);
    if (lane + o < 32) suf += y;
  }
  if (lane == 0 && above + suf < need_q) sh.cbin = -1;
  unsigned long long cum = above + (suf - own);  // mass of the bins above this lane's
#pragma unroll
  for (int i = 7; i >= 0; --i) {
    const unsigned long long nxt = cum + s8[i];
    if (cum < need_q && need_q <= nxt) {
      sh.cbin = 8 * lane + i;
      sh.cabove = cum;
      sh.ccount = bcnt[8 * lane + i];
    }
    cum = nxt;
  }
}

// keys: the P order keys (scores) in shared memory; mkey: kCovMaxCand 64-bit slots of
// shared memory (8-byte aligned); scratch: kSelScratchWords words of shared memory,
// 8-byte aligned (bin sums and counts at its start, the bitmap at kSelBitmapOff).
template <int NT, typename Bar>
__device__ inline void select_coverage(const uint32_t* keys, int P, int L, const kvq_select_params& prm,
                                       unsigned long long* mkey, uint32_t* scratch, int32_t* out, int32_t* cnt_out,
                                       int kmax, uint32_t* err, SelShared& sh, int tid, Bar& bar) {
  constexpr int NW = NT / 32;
  const int lane = tid & 31, warp = tid >> 5;
  const SelectSplit sp = select_split(P, prm);
  const int ns = sp.ns, rs = sp.rs, nC = sp.nC;
  auto is_cand = [&](int p) { return p >= ns && p < rs; };
  const int nwords = (P + 31) / 32;
  uint32_t* bs = scratch;                                                     // [3][256]
  int* bcnt = reinterpret_cast<int*>(scratch + 768);                          // [256]
  uint32_t* eqm = scratch + kCovEqOff;                                        // [nwords]
  uint32_t* chosen = scratch + kSelBitmapOff;
  // 1) largest finite score
  float hi = -INFINITY;
  for (int p = tid; p < P; p += NT)
    if (keys[p] != 0u) hi = fmaxf(hi, key_score(keys[p]));
#pragma unroll
  for (int o = 16; o; o >>= 1) hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  if (lane == 0) sh.wmax[warp] = hi;
  if (tid == 0) {
    sh.ckmin = ~0ull;
    sh.ckmax = 0ull;
  }
  bar();
  float smax = -INFINITY;
#pragma unroll
  for (int w = 0; w < NW; ++w) smax = fmaxf(smax, sh.wmax[w]);
  const double scale = static_cast<double>(prm.sm_scale);
  // 2) every page's mass once: the candidates' keys into mkey[p - ns], the totals, the
  //    candidates' key range
  double tot = 0.0, forced = 0.0;
  unsigned long long kmin = ~0ull, kmx = 0ull;
  for (int p = tid; p < P; p += NT) {
    const uint32_t k = keys[p];
    double m = 0.0;
    if (k != 0u && smax > -INFINITY) {
      const double n = p == P - 1 ? static_cast<double>(L - kPage * (P - 1)) : static_cast<double>(kPage);
      m = n * exp(scale * (static_cast<double>(key_score(k)) - static_cast<double>(smax)));
    }
    tot += m;
    if (is_cand(p)) {
      const unsigned long long mk = static_cast<unsigned long long>(__double_as_longlong(m));
      mkey[p - ns] = mk;
      kmin = min(kmin, mk);
      kmx = max(kmx, mk);
    } else {
      forced += m;
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmx = max(kmx, __shfl_xor_sync(0xffffffffu, kmx, o));
  }
  if (lane == 0) {
    atomicMin(&sh.ckmin, kmin);
    atomicMax(&sh.ckmax, kmx);
  }
  const double total = sel_block_sum<NT>(tot, sh, tid, bar);
  const double fsum = sel_block_sum<NT>(forced, sh, tid, bar);
  const double need = static_cast<double>(prm.coverage_ppm) * 1e-6 * total - fsum;
  // 3) the cut: every candidate whose key is above `prefix` in the bits >= shift, and the
  //    r lowest pages of those equal to it there (mode 1); none (0); all of positive mass (2)
  int mode = 0, shift = 0, r = 0;
  unsigned long long prefix = 0ull;
  if (need > 0.0 && nC > 0) {
    const unsigned long long need_q = __double2ull_ru(need * 0x1p46);  // >= 1 (2^kCovFixBits units)
    const unsigned long long lo = sh.ckmin, hk = sh.ckmax;
    shift = lo == hk ? 0 : 64 - __clzll(static_cast<long long>(lo ^ hk));  // bits below it are common
    prefix = hk;
    unsigned long long above = 0ull;
    int count = nC;
    mode = 1;
    while (shift > 0 && count > 1) {
      const int low = max(shift - 8, 0);
      const unsigned long long hm = shift >= 64 ? 0ull : (~0ull << shift);
      const unsigned long long want = prefix & hm;
      for (int i = tid; i < 1024; i += NT) scratch[i] = 0u;  // sum parts and counts
      bar();
      for (int i0 = warp * 32; i0 < nC; i0 += NT) {  // warp-uniform rounds of 32 candidates
        const int i = i0 + lane;
        int bin = -1;
        unsigned long long q = 0ull;
        if (i < nC) {
          const unsigned long long k = mkey[i];
          if ((k & hm) == want) {
            bin = static_cast<int>((k >> low) & ((1ull << (shift - low)) - 1ull));
            q = cov_fixed(k);
          }
        }
        const unsigned grp = __match_any_sync(0xffffffffu, bin);  // lanes of this lane's bin
        const unsigned leads = __ballot_sync(0xffffffffu, bin >= 0 && lane == __ffs(grp) - 1);
        if (__popc(leads) > 4) {  // spread over many bins: every lane adds its own (few conflicts)
          if (bin >= 0) {
            atomicAdd(&bs[bin], static_cast<unsigned>(q & 0x1FFFFull));
            atomicAdd(&bs[256 + bin], static_cast<unsigned>((q >> 17) & 0x1FFFFull));
            atomicAdd(&bs[512 + bin], static_cast<unsigned>(q >> 34));
            atomicAdd(&bcnt[bin], 1);
          }
        } else if (bin >= 0) {  // a few bins: one addition per bin, the group's sums reduced first
          const unsigned s0 = __reduce_add_sync(grp, static_cast<unsigned>(q & 0x1FFFFull));
          const unsigned s1 = __reduce_add_sync(grp, static_cast<unsigned>((q >> 17) & 0x1FFFFull));
          const unsigned s2 = __reduce_add_sync(grp, static_cast<unsigned>(q >> 34));
          if (lane == __ffs(grp) - 1) {
            atomicAdd(&bs[bin], s0);
            atomicAdd(&bs[256 + bin], s1);
            atomicAdd(&bs[512 + bin], s2);
            atomicAdd(&bcnt[bin], __popc(grp));
          }
        }
      }
      bar();
      if (warp == 0) cov_find_bin(bs, bcnt, above, need_q, sh, lane);
      bar();
      const int b = sh.cbin;
      if (b < 0) {  // even every candidate left does not reach the target: all of positive mass
        mode = 2;
        break;
      }
      prefix = want | (static_cast<unsigned long long>(b) << low);
      above = sh.cabove;
      count = sh.ccount;
      shift = low;  // (the next pass writes the bins and sh.c* only after two more barriers)
    }
    if (mode == 1) {
      if (count <= 1) {
        r = count;
      } else {  // `count` candidates of one exact mass: the fewest of them that reach the target
        const unsigned long long q = cov_fixed(prefix);
        const unsigned long long rq = q > 0ull ? (need_q - above + q - 1ull) / q : static_cast<unsigned long long>(count);
        r = rq < static_cast<unsigned long long>(count) ? static_cast<int>(rq) : count;
      }
    }
  }
  // 4) the bitmap: forced pages and the candidates above the cut (one ballot per word),
  //    and the candidates at the cut in eqm
  const unsigned long long hm = shift >= 64 ? 0ull : (~0ull << shift);
  const unsigned long long want = prefix & hm;
  for (int wd = warp; wd < nwords; wd += NW) {
    const int p = 32 * wd + lane;
    bool take = false, at = false;
    if (p < P) {
      if (!is_cand(p)) {
        take = true;
      } else if (mode == 2) {
        take = mkey[p - ns] != 0ull;
      } else if (mode == 1) {
        const unsigned long long k = mkey[p - ns] & hm;
        take = k > want;
        at = k == want;
      }
    }
    const unsigned tm = __ballot_sync(0xffffffffu, take), am = __ballot_sync(0xffffffffu, at);
    if (lane == 0) {
      chosen[wd] = tm;
      eqm[wd] = am;
    }
  }
  bar();
  if (mode == 1 && r > 0) {  // the r lowest pages at the cut (block scan over word ranges)
    const int WPT = (nwords + NT - 1) / NT;
    const int w_lo = min(nwords, tid * WPT), w_hi = min(nwords, w_lo + WPT);
    int eq = 0;
    for (int wd = w_lo; wd < w_hi; ++wd) eq += __popc(eqm[wd]);
    int tot_eq;
    int e = sel_exclusive_scan<NT>(eq, sh, &tot_eq, tid, bar);
    for (int wd = w_lo; wd < w_hi && e < r; ++wd) {
      unsigned m = eqm[wd], add = 0u;
      while (m && e < r) {
        const unsigned bit = m & (0u - m);
        add |= bit;
        m ^= bit;
        ++e;
      }
      chosen[wd] |= add;
    }
    bar();
  }
  emit_chosen<NT>(chosen, nwords, out, cnt_out, kmax, err, sh, tid, bar);
}

}  // namespace kvq
