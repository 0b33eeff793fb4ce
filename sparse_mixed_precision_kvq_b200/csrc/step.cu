// kvq_decode_step: one whole decode step -- append, page scores, top-k page selection and
// sparse attention with its log-sum-exp combine -- in a single persistent kernel.
//
// AMASS "decode-time sparse KV-cache attention for vLLM", "What is in the box": score
// every page from its resident summary, keep the best pages, attend only to those.  The
// arithmetic of every stage is the one of the separate calls (quant.cuh, score_tile.cuh,
// select_core.cuh, page_math.cuh); what changes is the schedule.
//
// Work units are (b, kv head) pairs u.  Each unit is cut into
//   score items:     32 ring slots of page summaries (1024 pages at D = 128),
//   attention items: 32 selected pages,
// and one queue orders all score items (unit by unit) before all attention items.
// One CTA per SM takes items from the queue (an atomic counter) until it runs dry.
//
// Inside a CTA, one producer warp takes the items and streams their bytes (summary rows,
// or the K and V chunks of selected pages) with bulk copies (TMA engine) into a ring of
// 8 KB shared-memory slots, each with a "full" and an "empty" mbarrier.  It holds two
// items: while the current one is issued into the ring, the next one is already resolved
// (its page list read) and its whole byte range requested into L2.  Eight consumer warps take the slots round-robin:
// slot k of the CTA's stream goes to consumer k mod 8, and every item is padded to a
// multiple of 8 slots, so each consumer sees the same number of slots of every item and
// all of them reach the item's end together.  At an item's end the consumers meet at a
// named barrier of their own while the producer keeps streaming the next item.
//
//  - score item: each consumer scores the summaries of its slots (tensor-core tile) and
//    writes them to `scores`; the consumer whose slot holds the page of the appended token
//    first writes the token (quantised) and the new summary row, patching the row in the
//    slot.  The CTA then counts the item on the unit; the CTA that finishes the unit's last
//    score item selects its pages (select_core.cuh, over the unit's scores read back
//    from L2) and marks the unit ready (counter + 1).
//  - attention item: the producer waits until the unit is ready, reads the chosen pages
//    and their block-table entries (one lane per page), and streams the pages; consumers
//    run the online-softmax page math; the CTA merges its eight warp partials, and either
//    writes the output (a unit with one attention item) or stores a partial and counts
//    the item on the unit; the last CTA to arrive merges the unit's partials.
//
// No wait can deadlock: every score item is taken before any attention item, score items
// never wait, so the units an attention item waits for are always being finished by CTAs
// that are running.  Every wait is bounded (2 s, or the limit the workspace sets); on a timeout the CTA flags
// KVQ_DERR_TIMEOUT, stops issuing copies, waits (bounded) for the copies in flight and
// leaves.  Counters are returned to zero by the CTA that last uses them.
#include <math.h>

#include "kvq_internal.cuh"
#include "page_math.cuh"
#include "ptx.cuh"
#include "quant.cuh"
#include "score_tile.cuh"
#include "select_core.cuh"

namespace kvq {
namespace {

constexpr int kCW = 8;                        // consumer warps
constexpr int kCT = kCW * 32;                 // consumer threads
constexpr int kStepThreads = kCT + 32;        // + the producer warp
constexpr int kSlot = 8192;                   // ring slot bytes: one 16-bit page (K + V) at D = 128
// Item sizes: large enough to amortise an item's fixed costs (a few dependent memory
// round trips and consumer barriers), small enough to spread over the CTAs.
constexpr int kASlots = 32;                   // score item: ring slots of summaries (1024 at D = 128)
constexpr int kBPages = 32;                   // attention item: selected pages (one producer lane each)
constexpr int kBMax = kBPages;
constexpr int kMaxRingSlots = 24;             // data slots (a multiple of kCW: each warp owns slots w, w + 8, ...)
constexpr int kNDesc = 64;                    // descriptor ring (a multiple of kCW, a power of two)
constexpr int kMaxSmem = 232448 - 4096;       // 227 KB per CTA, less the static shared memory
constexpr int kCtlWords = 16;                 // [0] item queue, [1] CTAs finished, then a_done, b_done
static_assert(kBMax <= 32, "one producer lane per page of an attention item");

enum : int { KIND_A = 0, KIND_B = 1, KIND_END = 2 };

// One position of the CTA's stream: what to copy into the ring and what it holds.
struct SlotDesc {
  int kind;
  int unit;   // b * Hkv + g
  int item;   // score item index, or attention item index (= its partial slot)
  int p;      // score: first page of the slot; attention: page index
  int n;      // score: pages in the slot (0: padding); attention: tier (-1: padding)
  int nv;     // attention: valid tokens of the page
  int last;   // last position of the item for the consumer that takes it
  int bytes;  // bytes to copy (0: nothing)
  const void* src;
};

struct StepArgs {
  DevCache c;
  const int32_t* pos;  // nullable: no append
  const uint16_t* k_new;
  const uint16_t* v_new;
  const uint16_t* q;
  kvq_select_params prm;
  float* scores;
  int32_t* sel;
  int32_t* cnt;
  int kmax;
  float scale_log2;
  uint16_t* out;
  float* lse;
  unsigned* ctl;     // [0] item queue, [1] CTAs finished
  unsigned* a_done;  // [U] score items finished (+1 once the unit's pages are chosen)
  unsigned* b_done;  // [U] attention items finished
  float* part_o;     // [attention items][G][D]
  float* part_ml;    // [attention items][G][2]
  int ns;            // ring slots
  int union_bytes;   // keys + histogram of the selection / warp partials of the merge
  int keys_bytes;    // selection keys (the histogram follows them)
};

template <int D>
struct SummariesPerSlot {
  static constexpr int value = kSlot / (2 * D);
};

__host__ __device__ inline int pages_of(int L, int max_pages) {
  const int P = (max(L, 0) + kPage - 1) / kPage;
  return P < max_pages ? P : max_pages;
}
// Score items of a unit of P pages with items of up to `as` slots (balanced split).
template <int D>
__host__ __device__ inline int score_items(int P, int as) {
  const int nsl = (P + SummariesPerSlot<D>::value - 1) / SummariesPerSlot<D>::value;
  return nsl > 0 ? (nsl + as - 1) / as : 1;
}
// Pages attended for a unit of P pages (the selection's count, clamped to kmax).
__host__ __device__ inline int attn_pages(int P, const kvq_select_params& prm, int kmax) {
  return min(select_split(P, prm).count(P), kmax);
}
__host__ __device__ inline int attn_items(int P, const kvq_select_params& prm, int kmax, int bs) {
  const int n = attn_pages(P, prm, kmax);
  return n > 0 ? (n + bs - 1) / bs : 1;
}


// last b with tab[b] <= i (tab strictly increasing, tab[0] = 0)
__device__ inline int find_b(const int* tab, int B, int i) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tab[mid] <= i) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Bounded mbarrier wait (a spin on test_wait: no suspension, so no late wake-up) that
// gives up at once when the CTA has given up (*abort), and makes the CTA give up when the
// time runs out.
__device__ inline bool wait_or_abort(uint32_t bar, uint32_t parity, volatile int* abort, unsigned long long limit_ns) {
  if (mbar_test_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  while (!mbar_test_wait(bar, parity)) {
    if (*abort) return false;
    if (globaltimer() - t0 > limit_ns) {
      *abort = 1;
      return false;
    }
  }
  return true;
}

// Barrier of the eight consumer warps (named barrier 1; the producer never joins it).
// It returns false, in every consumer alike, once the CTA has given up: the OR of the
// abort flag is taken by the barrier itself, so all warps leave their loops together and
// no warp is ever left waiting at a barrier the others skip.  Every wait before a barrier
// is bounded, so every barrier completes.
struct ConsumerBar {
  volatile int* abort;
  __device__ inline bool operator()() { return !bar_sync_or(1, kCT, *abort != 0); }
};

// Merge of the kCW warp partials in shared memory (o [G][D] then (m, l) [G][2] per warp)
// for element (h, d): M = max m_w, L = sum l_w 2^(m_w - M), o = sum o_w 2^(m_w - M).
template <int D>
__device__ inline void merge_warps(const float* wp, int G, int h, int d, float& M, float& Ls, float& o) {
  const int stride = G * (D + 2);
  float mv[kCW], lv[kCW], ov[kCW];
#pragma unroll
  for (int w = 0; w < kCW; ++w) {
    ov[w] = wp[w * stride + h * D + d];
    mv[w] = wp[w * stride + G * D + 2 * h];
    lv[w] = wp[w * stride + G * D + 2 * h + 1];
  }
  M = -INFINITY;
#pragma unroll
  for (int w = 0; w < kCW; ++w) M = fmaxf(M, mv[w]);
  o = 0.f;
  Ls = 0.f;
  if (M != -INFINITY) {
#pragma unroll
    for (int w = 0; w < kCW; ++w) {
      const float f = mv[w] == -INFINITY ? 0.f : exp2f(mv[w] - M);
      o += ov[w] * f;
      Ls += lv[w] * f;
    }
  }
}

template <bool BF16>
__device__ inline void write_out(uint16_t* out, float* lse, size_t row, int d, int D, float M, float Ls, float o) {
  const bool any = !(Ls <= 0.f);  // a NaN sum (a NaN key or value) gives a NaN output
  const float r = any ? o / Ls : 0.f;
  if constexpr (BF16) out[row * D + d] = __bfloat16_as_ushort(__float2bfloat16_rn(r));
  else out[row * D + d] = __half_as_ushort(__float2half_rn(r));
  if (d == 0 && lse != nullptr) lse[row] = any ? (M + log2f(Ls)) * 0.69314718055994531f : -INFINITY;
}

template <int D, bool BF16>
__global__ void __launch_bounds__(kStepThreads, 1) step_kernel(StepArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const DevCache& c = a.c;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ns = a.ns;
  const int B = c.B, Hkv = c.Hkv, G = c.G;
  constexpr int SP = SummariesPerSlot<D>::value;

  unsigned char* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)ns * kSlot);  // [ns] data landed
  uint64_t* dfull = full + ns;                                              // [kNDesc] descriptor written
  uint64_t* dempty = dfull + kNDesc;                                        // [kNDesc] position consumed
  SlotDesc* desc = reinterpret_cast<SlotDesc*>(dempty + kNDesc);            // [kNDesc]
  unsigned char* un = reinterpret_cast<unsigned char*>(desc + kNDesc);
  int* tabA = reinterpret_cast<int*>(un + a.union_bytes);  // [B + 1] first score item of b
  int* tabB = tabA + B + 1;                                  // [B + 1] first attention item of b
  int* tabL = tabB + B + 1;                                  // [B] sequence lengths
  __shared__ SelShared sel_sh;
  __shared__ int s_abort, s_flag;
  __shared__ int s_scan[2][kStepThreads / 32 + 1];

  if (tid == 0) {
    for (int i = 0; i < ns; ++i) mbar_init(smem_u32(&full[i]), 1);
    for (int i = 0; i < kNDesc; ++i) {
      mbar_init(smem_u32(&dfull[i]), 1);
      mbar_init(smem_u32(&dempty[i]), 1);
    }
    s_abort = 0;
    s_flag = 0;
    mbar_init_fence();
  }
  griddep_wait();  // the cache and the inputs come from earlier work on the stream
  const unsigned long long wait_ns = wait_limit_ns(a.ctl, kWaitLimitWord);

  // item tables: exclusive prefix sums over b of the items of b's Hkv units
  constexpr int as = kASlots, bs = kBPages;
  {
    constexpr int NW = kStepThreads / 32;
    const int per = (B + kStepThreads - 1) / kStepThreads;
    const int lo = min(B, tid * per), hi = min(B, lo + per);
    int sa = 0, sb = 0;
    for (int b = lo; b < hi; ++b) {
      const int L = max(c.seq_len[b], 0);
      tabL[b] = L;
      const int P = pages_of(L, c.max_pages);
      sa += score_items<D>(P, as) * Hkv;
      sb += attn_items(P, a.prm, a.kmax, bs) * Hkv;
    }
    int x = sa, y = sb;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int xa = __shfl_up_sync(0xffffffffu, x, o), yb = __shfl_up_sync(0xffffffffu, y, o);
      if (lane >= o) {
        x += xa;
        y += yb;
      }
    }
    if (lane == 31) {
      s_scan[0][warp] = x;
      s_scan[1][warp] = y;
    }
    __syncthreads();
    if (tid == 0) {
      int ra = 0, rb = 0;
      for (int w = 0; w < NW; ++w) {
        const int ta = s_scan[0][w], tb = s_scan[1][w];
        s_scan[0][w] = ra;
        s_scan[1][w] = rb;
        ra += ta;
        rb += tb;
      }
      s_scan[0][NW] = ra;
      s_scan[1][NW] = rb;
    }
    __syncthreads();
    int ra = s_scan[0][warp] + x - sa, rb = s_scan[1][warp] + y - sb;
    for (int b = lo; b < hi; ++b) {
      tabA[b] = ra;
      tabB[b] = rb;
      const int P = pages_of(tabL[b], c.max_pages);
      ra += score_items<D>(P, as) * Hkv;
      rb += attn_items(P, a.prm, a.kmax, bs) * Hkv;
    }
    if (tid == 0) {
      tabA[B] = s_scan[0][NW];
      tabB[B] = s_scan[1][NW];
    }
    __syncthreads();
  }
  const int totA = tabA[B], totB = tabB[B];

  if (warp == kCW) {
    // ------------------------------------------------------------------ producer warp
    // Two items in hand: `cur` being issued into the ring, `nxt` already taken from the
    // queue and, as soon as it can be, resolved (its page list read) and requested into L2,
    // so that its bytes stream while the ring still drains `cur`.
    struct Item {
      int valid, kind, u, b, g, item, resolved;
      int p0, np, S;  // score: first page, pages, slots (padded); attention: pages, slots
      // attention: lane l holds page l of the item
      const unsigned char* psrc;
      int tier, nv, pg;
    };
    int k = 0;  // positions published
    bool failed = false;
    // Write the descriptors of stream positions k .. k + n - 1 (n <= 32), lane i the one
    // of position k + i, each once the consumer of position k + i - kNDesc is done with
    // its entry.  The copies themselves are issued by the consumer warps that own the
    // positions: bulk copies issued by one warp alone do not keep HBM busy.
    auto publish = [&](const SlotDesc& d, int n) -> bool {
      bool ok = true;
      if (lane < n) {
        const int kk = k + lane;
        const int e = kk & (kNDesc - 1);
        ok = wait_or_abort(smem_u32(&dempty[e]), ((kk / kNDesc) & 1) ^ 1, &s_abort, wait_ns);
        if (ok) {
          desc[e] = d;
          mbar_arrive(smem_u32(&dfull[e]));
        }
      }
      ok = __all_sync(0xffffffffu, ok);
      k += n;
      return ok;
    };
    // Take the next item from the queue (no waiting).
    auto take = [&](Item& it) {
      int item = 0;
      if (lane == 0) item = static_cast<int>(atomicAdd(&a.ctl[0], 1u));
      item = __shfl_sync(0xffffffffu, item, 0);
      it.valid = item < totA + totB;
      it.resolved = 0;
      if (!it.valid) return;
      if (item < totA) {
        const int b = find_b(tabA, B, item);
        const int P = pages_of(tabL[b], c.max_pages);
        const int na = score_items<D>(P, as);
        const int r = item - tabA[b], j = r % na;
        it.kind = KIND_A;
        it.b = b;
        it.g = r / na;
        it.p0 = j * as * SP;
        it.np = min(P, it.p0 + as * SP) - it.p0;
        it.item = item;
      } else {
        const int ib = item - totA;
        const int b = find_b(tabB, B, ib);
        const int P = pages_of(tabL[b], c.max_pages);
        const int n = attn_pages(P, a.prm, a.kmax);
        const int nb = attn_items(P, a.prm, a.kmax, bs);
        const int r = ib - tabB[b], j = r % nb;
        it.kind = KIND_B;
        it.b = b;
        it.g = r / nb;
        it.p0 = j * bs;                          // first rank
        it.np = max(0, min(n, it.p0 + bs) - it.p0);
        it.item = ib;
      }
      it.u = it.b * Hkv + it.g;
    };
    // Read the item's page list and ask L2 for its bytes.  An attention item needs its unit's
    // pages chosen first: with `block` the producer waits for that (bounded), otherwise it
    // returns false when they are not chosen yet.
    auto resolve = [&](Item& it, bool block) -> bool {
      const int L = tabL[it.b];
      const int P = pages_of(L, c.max_pages);
      if (it.kind == KIND_A) {
        const int nsl = (it.np + SP - 1) / SP;
        it.S = max(kCW, (nsl + kCW - 1) / kCW * kCW);
        const uint16_t* src = c.summary + ((size_t)it.u * c.max_pages + it.p0) * D;
        for (int s = lane; s < nsl; s += 32)
          bulk_prefetch_l2(src + (size_t)s * SP * D, (uint32_t)min(SP, it.np - s * SP) * D * 2);
        it.resolved = 1;
        return true;
      }
      // wait until the unit's pages are chosen (a_done = score items + 1)
      const unsigned target = static_cast<unsigned>(score_items<D>(P, as)) + 1u;
      int ok = 1;
      if (lane == 0) {
        if (ld_acquire_gpu(&a.a_done[it.u]) < target) {
          ok = 0;
          if (block) {
            const unsigned long long t0 = globaltimer();
            for (;;) {
              __nanosleep(64);
              if (ld_acquire_gpu(&a.a_done[it.u]) >= target) {
                ok = 1;
                break;
              }
              if (*reinterpret_cast<volatile int*>(&s_abort) || globaltimer() - t0 > wait_ns) {
                ok = -1;
                break;
              }
            }
          }
        }
        if (ok == 1) fence_proxy_async_global();  // the pages may have been written by another CTA
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (ok < 0) failed = true;
      if (ok <= 0) return false;
      const int n = min(max(__ldcg(&a.cnt[it.u]), 0), a.kmax);
      it.np = max(0, min(n, it.p0 + it.np) - it.p0);  // the selection's own count (equal but for errors)
      it.S = max(kCW, (it.np + kCW - 1) / kCW * kCW);
      it.psrc = nullptr;
      it.tier = -1;
      it.nv = 0;
      it.pg = -1;
      if (lane < it.np) {
        const int p = __ldcg(&a.sel[(size_t)it.u * a.kmax + it.p0 + lane]);
        it.pg = p;
        if (p >= 0 && p < P) {
          const unsigned char *s_, *v_;
          int tier;
          if (page_chunks(c, it.b, p, it.g, tier, s_, v_)) {
            it.psrc = s_;
            it.tier = tier;
            it.nv = min(kPage, L - p * kPage);
            bulk_prefetch_l2(s_, 2u * c.chunk[tier]);
          }
        } else {
          set_err(c.err, KVQ_DERR_BAD_PAGE);
        }
      }
      it.resolved = 1;
      return true;
    };
    // Publish all positions of `it` (lane s: positions s, s + 32, ... of the item).
    auto issue = [&](const Item& it) {
      for (int s0 = 0; s0 < it.S && !failed; s0 += 32) {
        const int s = s0 + lane;
        SlotDesc d;
        if (it.kind == KIND_A) {
          const int n = s * SP < it.np ? min(SP, it.np - s * SP) : 0;
          d = SlotDesc{KIND_A, it.u, it.item, it.p0 + s * SP, n, 0, s >= it.S - kCW ? 1 : 0, n * D * 2,
                       c.summary + ((size_t)it.u * c.max_pages + it.p0 + (size_t)s * SP) * D};
        } else {
          const bool real = s < it.np && it.tier >= 0;
          d = SlotDesc{KIND_B, it.u, it.item, it.pg, real ? it.tier : -1, it.nv, s >= it.S - kCW ? 1 : 0,
                       real ? 2 * c.chunk[it.tier] : 0, it.psrc};
        }
        failed = !publish(d, min(32, it.S - s0));
      }
    };

    Item cur, nxt;
    take(cur);
    if (cur.valid) resolve(cur, true);
    while (cur.valid && !failed) {
      take(nxt);
      if (nxt.valid) resolve(nxt, false);
      issue(cur);
      if (nxt.valid && !nxt.resolved && !failed) resolve(nxt, true);
      cur = nxt;
    }
    if (!failed) failed = !publish(SlotDesc{KIND_END, 0, 0, 0, 0, 0, 1, 0, nullptr}, kCW);
    if (failed && lane == 0) {
      s_abort = 1;
      set_err(c.err, KVQ_DERR_TIMEOUT);
    }
  } else {
    // ---------------------------------------------------------------- consumer warps
    ConsumerBar cb{&s_abort};
    // This warp takes stream positions k = warp + m * kCW (m = 0, 1, ...); position k lands
    // in data slot k % ns, one of the ns / kCW slots the warp owns, and the warp issues the
    // copy of each of its positions itself, as soon as its descriptor is written and its
    // slot is free, keeping up to ns / kCW of them in flight.
    const int R = ns / kCW;
    int m = 0;   // positions consumed
    int mi = 0;  // positions whose copy has been issued
    bool end_issued = false;
    // Issue the copies of the next positions whose descriptors are there (without
    // waiting), or, with `need`, first wait for position m's descriptor.
    auto top_up = [&](bool need) -> bool {
      while (!end_issued && mi < m + R) {
        const int k = warp + mi * kCW;
        const int e = k & (kNDesc - 1);
        const uint32_t par = (k / kNDesc) & 1;
        bool have;
        if (need && mi == m) {
          have = wait_or_abort(smem_u32(&dfull[e]), par, &s_abort, wait_ns);
          if (!have) return false;
        } else {
          have = mbar_test_wait(smem_u32(&dfull[e]), par);
          if (!have) break;
        }
        const SlotDesc& d = desc[e];
        const int slot = k % ns;
        if (lane == 0) {
          const uint32_t fb = smem_u32(&full[slot]);
          if (d.bytes > 0) {
            mbar_expect_tx(fb, static_cast<uint32_t>(d.bytes));
            bulk_copy_g2s(smem_u32(ring + (size_t)slot * kSlot), d.src, static_cast<uint32_t>(d.bytes), fb);
          } else {
            mbar_arrive(fb);
          }
        }
        end_issued = d.kind == KIND_END;
        ++mi;
      }
      return true;
    };
    auto wait_slot = [&](int& slot, SlotDesc& d) -> bool {
      if (!top_up(true)) return false;
      const int k = warp + m * kCW;
      slot = k % ns;
      if (!wait_or_abort(smem_u32(&full[slot]), (k / ns) & 1, &s_abort, wait_ns)) return false;
      d = desc[k & (kNDesc - 1)];
      return true;
    };
    auto release_slot = [&](int slot) {
      (void)slot;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&dempty[(warp + m * kCW) & (kNDesc - 1)]));
      ++m;
      top_up(false);  // the slot just freed takes the warp's next position
    };

    // The CTA chooses unit u's pages (all consumer threads).
    auto select_unit = [&](int u, int P) -> bool {
      uint32_t* keys = reinterpret_cast<uint32_t*>(un);
      const float* sc = a.scores + (size_t)u * c.max_pages;
      bool nan_seen = false;
      for (int p0 = tid; p0 < P; p0 += 4 * kCT) {  // four loads in flight per thread
        float v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) v[j] = p0 + j * kCT < P ? __ldcg(sc + p0 + j * kCT) : 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (p0 + j * kCT < P) keys[p0 + j * kCT] = order_key(v[j], nan_seen);
      }
      if (nan_seen) set_err(c.err, KVQ_DERR_NAN_SCORE);
      if (!cb()) return false;
      select_pages<kCT>(keys, P, a.prm, a.sel + (size_t)u * a.kmax, a.cnt + u, a.kmax, c.err,
                        reinterpret_cast<uint32_t*>(un + a.keys_bytes), sel_sh, tid, cb);
      if (!cb()) return false;
      if (tid == 0) {  // the barrier orders every thread's sel/cnt writes before this fence
        __threadfence();
        atomicAdd(&a.a_done[u], 1u);  // ready
      }
      return true;
    };

    auto score_item = [&](int slot, SlotDesc d) -> bool {
      const int u = d.unit, b = u / Hkv, g = u % Hkv;
      const int P = pages_of(tabL[b], c.max_pages);
      QFrag<D, BF16> qf;
      bool bad = false;
      qf.load(a.q, c.Hq, G, b, g, lane, bad);
      int pa = -1;  // position of the token appended to this unit
      if (a.pos != nullptr) {
        const int ps = a.pos[b];
        if (ps >= 0) {
          if (ps < c.max_pages * kPage && ps / kPage < P) pa = ps;
          else if (lane == 0 && d.p == 0) set_err(c.err, KVQ_DERR_BAD_POS);
        }
      }
      float* srow = a.scores + (size_t)u * c.max_pages;
      for (;;) {
        if (d.n > 0) {
          uint16_t* rows = reinterpret_cast<uint16_t*>(ring + (size_t)slot * kSlot);
          const int pg = pa / kPage;
          if (pa >= 0 && pg >= d.p && pg < d.p + d.n) {
            append_token_warp<BF16>(c, b, g, pa, a.k_new + (size_t)u * D, a.v_new + (size_t)u * D, lane,
                                    rows + (size_t)(pg - d.p) * D);
            __threadfence();
            fence_proxy_async_global();
            fence_proxy_async();
            __syncwarp();
          }
          for (int t = 0; t < d.n; t += 16) {
            uint4 av[2][D / 32];
            load_tile_rows<D>(rows + (size_t)t * D, lane, av);
            float m0, m1;
            tile_scores<D, BF16>(av, qf, G, lane, m0, m1);
            if ((lane & 3) == 0) {
              const int r0 = t + (lane >> 2), r1 = r0 + 8;
              if (r0 < d.n) srow[d.p + r0] = m0;
              if (r1 < d.n) srow[d.p + r1] = m1;
            }
          }
        }
        const int last = d.last;
        release_slot(slot);
        if (last || !wait_slot(slot, d)) break;  // a failed wait: the barrier below reports it to all
      }
      if (bad) set_err(c.err, KVQ_DERR_FP16_RANGE);
      if (!cb()) return false;
      if (tid == 0) {  // the barrier orders every warp's score writes before this fence
        __threadfence();
        const unsigned old = atomicAdd(&a.a_done[u], 1u);
        s_flag = (old + 1u == static_cast<unsigned>(score_items<D>(P, as))) ? 1 : 0;
      }
      if (!cb()) return false;
      if (s_flag) {
        __threadfence();
        return select_unit(u, P);
      }
      return true;
    };

    auto attn_item = [&](int slot, SlotDesc d) -> bool {
      const int u = d.unit, b = u / Hkv, g = u % Hkv;
      const int ib = d.item;
      WarpState<D> st;
      begin_segment<D, BF16>(a.q, c.Hq, G, b, g, lane, st);
      for (;;) {
        if (d.n >= 0)
          process_page<D, BF16>(ring + (size_t)slot * kSlot, d.n, d.nv, lane, a.scale_log2, st);
        const int last = d.last;
        release_slot(slot);
        if (last || !wait_slot(slot, d)) break;  // a failed wait: the barrier below reports it to all
      }
      float* wp = reinterpret_cast<float*>(un);
      float* mine = wp + (size_t)warp * G * (D + 2);
      write_warp_partial<D>(G, st, mine, mine + G * D, lane);
      if (!cb()) return false;
      const int P = pages_of(tabL[b], c.max_pages);
      const int nb = attn_items(P, a.prm, a.kmax, bs);
      const size_t row0 = (size_t)b * c.Hq + (size_t)g * G;
      for (int e = tid; e < G * D; e += kCT) {
        const int h = e / D, dd = e % D;
        float M, Ls, o;
        merge_warps<D>(wp, G, h, dd, M, Ls, o);
        if (nb == 1) {
          write_out<BF16>(a.out, a.lse, row0 + h, dd, D, M, Ls, o);
        } else {
          a.part_o[((size_t)ib * G + h) * D + dd] = o;
          if (dd == 0) {
            a.part_ml[((size_t)ib * G + h) * 2] = M;
            a.part_ml[((size_t)ib * G + h) * 2 + 1] = Ls;
          }
        }
      }
      if (nb == 1) {
        if (tid == 0) a.a_done[u] = 0u;  // the unit is finished: its counter is free again
      } else {
        if (!cb()) return false;
        if (tid == 0) {  // the barrier orders every thread's partial writes before this fence
          __threadfence();
          const unsigned old = atomicAdd(&a.b_done[u], 1u);
          s_flag = (old + 1u == static_cast<unsigned>(nb)) ? 1 : 0;
        }
        if (!cb()) return false;
        if (s_flag) {  // the unit's last attention item: merge its partials into the output
          __threadfence();
          const int first = tabB[b] + g * nb;
          for (int e = tid; e < G * D; e += kCT) {
            const int h = e / D, dd = e % D;
            float M = -INFINITY, o = 0.f, Ls = 0.f;
            for (int j0 = 0; j0 < nb; j0 += 8) {
              float mv[8], lv[8], ov[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                mv[i] = -INFINITY;
                lv[i] = 0.f;
                ov[i] = 0.f;
                if (j0 + i < nb) {
                  const size_t s = (size_t)first + j0 + i;
                  const float2 ml = __ldcg(reinterpret_cast<const float2*>(&a.part_ml[(s * G + h) * 2]));
                  mv[i] = ml.x;
                  lv[i] = ml.y;
                  ov[i] = __ldcg(&a.part_o[(s * G + h) * D + dd]);
                }
              }
              float Mn = M;
#pragma unroll
              for (int i = 0; i < 8; ++i) Mn = fmaxf(Mn, mv[i]);
              if (Mn == -INFINITY) continue;
              const float rs = M == -INFINITY ? 0.f : exp2f(M - Mn);
              o *= rs;
              Ls *= rs;
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float f = mv[i] == -INFINITY ? 0.f : exp2f(mv[i] - Mn);
                o += ov[i] * f;
                Ls += lv[i] * f;
              }
              M = Mn;
            }
            write_out<BF16>(a.out, a.lse, row0 + h, dd, D, M, Ls, o);
          }
          if (tid == 0) {
            a.a_done[u] = 0u;
            a.b_done[u] = 0u;
          }
        }
      }
      return cb();  // the partial area is free for the next item
    };

    // Every consumer warp passes the same sequence of consumer barriers: items end with
    // barriers that all of them reach, and leaving the loop (end of the stream, or a failed
    // wait for the first slot of an item) costs one barrier too -- the one the other warps
    // reach at the end of that item when the CTA has given up.
    for (;;) {
      int slot;
      SlotDesc d;
      if (!wait_slot(slot, d) || d.kind == KIND_END) {
        cb();
        break;
      }
      const bool ok = d.kind == KIND_A ? score_item(slot, d) : attn_item(slot, d);
      if (!ok) break;
    }
    if (*reinterpret_cast<volatile int*>(&s_abort) && lane == 0) {
      set_err(c.err, KVQ_DERR_TIMEOUT);
      // let this warp's copies still in flight land before the CTA leaves (bounded)
      for (int j = m; j < mi; ++j) {
        const int k = warp + j * kCW;
        mbar_wait_bounded(smem_u32(&full[k % ns]), (k / ns) & 1, wait_ns);
      }
    }
  }

  __syncthreads();
  if (tid == 0) {  // the last CTA out returns the queue to zero for the next call
    __threadfence();
    const unsigned old = atomicAdd(&a.ctl[1], 1u);
    if (old + 1u == gridDim.x) {
      a.ctl[0] = 0u;
      a.ctl[1] = 0u;
      __threadfence();
    }
  }
  griddep_launch_dependents();
}

// Shared-memory plan of a launch: ring slots and the size of the keys / partials area.
struct StepPlan {
  int ns;
  int union_bytes;
  int keys_bytes;
  size_t smem;
};

inline StepPlan step_plan(const DevCache& c) {
  StepPlan pl;
  pl.keys_bytes = (int)(((size_t)c.max_pages * 4 + 15) / 16 * 16);
  const size_t sel = (size_t)pl.keys_bytes + kSelScratchWords * 4;
  const size_t parts = (size_t)kCW * c.G * (c.D + 2) * 4;
  pl.union_bytes = (int)(((sel > parts ? sel : parts) + 15) / 16 * 16);
  const size_t tables = ((size_t)3 * c.B + 2) * 4;
  const size_t fixed = (size_t)pl.union_bytes + tables + kNDesc * (2 * 8 + sizeof(SlotDesc));
  const size_t per_slot = kSlot + 8;
  long long ns = fixed < (size_t)kMaxSmem ? (long long)((kMaxSmem - fixed) / per_slot) : 0;
  if (ns > kMaxRingSlots) ns = kMaxRingSlots;
  ns = ns / kCW * kCW;
  pl.ns = (int)ns;
  pl.smem = (size_t)pl.ns * per_slot + fixed;
  return pl;
}

template <int D, bool BF16>
cudaError_t launch_step_d(const StepArgs& a, int num_ctas, size_t smem, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(step_kernel<D, BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(step_kernel<D, BF16>, dim3(num_ctas), dim3(kStepThreads), smem, s, a);
}

size_t attn_items_bound(const DevCache& c, int kmax) {
  const size_t per_unit = (size_t)((kmax + kBPages - 1) / kBPages);
  return (size_t)c.B * c.Hkv * (per_unit > 0 ? per_unit : 1);
}

}  // namespace

bool step_supported(const DevCache& c) {
  if (c.host_tiers != 0) return false;  // its pages are fetched by bulk copies only
  for (int t = 0; t < kNumTiers; ++t)
    if (c.vpool[t] != nullptr) return false;  // ... of adjacent K and V chunks
  if ((long long)c.B * c.Hkv * 2 + kCtlWords > (long long)kWaitLimitWord) return false;
  return step_plan(c).ns >= kCW;
}

// Workspace: [kCounterBytes] control words (queue, CTAs finished, per-unit score and
// attention arrivals; zero between calls), then the attention partials
// ([items][G][D] o, [items][G][2] (m, l)).
size_t step_workspace_bytes(const DevCache& c, int kmax) {
  return kCounterBytes + attn_items_bound(c, kmax) * c.G * ((size_t)c.D + 2) * sizeof(float);
}

cudaError_t launch_step(const DevCache& c, const int32_t* pos, const void* k_new, const void* v_new,
                        const void* q, const kvq_select_params& prm, float* scores, int32_t* sel, int32_t* cnt,
                        int kmax, float sm_scale, void* out, float* lse, void* ws, int num_ctas, cudaStream_t s) {
  StepArgs a;
  a.c = c;
  a.pos = pos;
  a.k_new = static_cast<const uint16_t*>(k_new);
  a.v_new = static_cast<const uint16_t*>(v_new);
  a.q = static_cast<const uint16_t*>(q);
  a.prm = prm;
  a.scores = scores;
  a.sel = sel;
  a.cnt = cnt;
  a.kmax = kmax;
  a.scale_log2 = sm_scale * 1.4426950408889634f;
  a.out = static_cast<uint16_t*>(out);
  a.lse = lse;
  unsigned* w = static_cast<unsigned*>(ws);
  const size_t U = (size_t)c.B * c.Hkv;
  a.ctl = w;
  a.a_done = w + kCtlWords;
  a.b_done = a.a_done + U;
  a.part_o = reinterpret_cast<float*>(static_cast<unsigned char*>(ws) + kCounterBytes);
  a.part_ml = a.part_o + attn_items_bound(c, kmax) * c.G * c.D;
  const StepPlan pl = step_plan(c);
  a.ns = pl.ns;
  a.union_bytes = pl.union_bytes;
  a.keys_bytes = pl.keys_bytes;
  const bool bf = c.dtype == KVQ_DT_BF16;
  if (c.D == 128) return bf ? launch_step_d<128, true>(a, num_ctas, pl.smem, s) : launch_step_d<128, false>(a, num_ctas, pl.smem, s);
  if (c.D == 64) return bf ? launch_step_d<64, true>(a, num_ctas, pl.smem, s) : launch_step_d<64, false>(a, num_ctas, pl.smem, s);
  return cudaErrorInvalidValue;
}

}  // namespace kvq
