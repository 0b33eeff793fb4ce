// kvq_sparse_decode_attn: attention over the selected pages only, split-K over CTAs,
// followed by a log-sum-exp combine.
//
// AMASS "decode-time sparse KV-cache attention for vLLM", "What is in the box": a sparse
// paged kernel reads just the selected pages.  ARGUS "Virtual Memory for Transformers",
// "Why It Works: Storage vs. Computation": low-bit pages are turned back into high
// precision before attention; no low-bit arithmetic enters the softmax.
//
// Work split.  The selected pages of all (b, g) are one flat list (segment bg holds
// cnt[bg] pages); every warp of the grid (one CTA per SM, 8 warps each) is an
// independent worker u that takes the contiguous slice [u*W, (u+1)*W),
// W = ceil(total / #workers), so every warp reads the same number of pages whatever the
// per-sequence lengths are.  A warp looks up the chunk addresses of up to 32 upcoming
// pages at once (one per lane) and runs its own copy pipeline: lane 0 issues one bulk
// copy (cp.async.bulk, TMA engine) per page (K and V chunks are adjacent) into the
// warp's shared-memory ring, completion on an mbarrier.  No CTA-wide barrier is needed
// between the prologue and the end of the CTA's pages.
//
// Math per page (16 tokens, the kv head's G <= 8 query heads), warp-level tensor-core
// mma m16n8k16 with fp32 accumulation:
//   S^T[t][h] = K[t][:] . q[h][:]      A = K rows (tokens), B = q^T (heads as N)
//   O^T[d][h] += V^T[d][:] . P^T[:][h] A = V^T rows (channels), B = P^T via movmatrix
// The page byte order is the mma operand order, so every operand is one 16-byte
// conflict-free shared-memory load per lane.  Quantised pages: codes are converted
// exactly to centred 16-bit floats c - 2^(b-1) in registers (magic-exponent bit tricks)
// and the per-group affine map is applied around the mma with z' = zero + 2^(b-1)*scale:
// for K, S += scale_t * (codes . q) + z'_t * sum(q over the group); for V, P^T is scaled
// per token by the group's scale before the mma and sum_t z'_t * p_t is accumulated on
// the side.  P^T enters the tensor core as a 16-bit hi + lo pair (two mmas), so the only
// 16-bit rounding on the way to the output is the final cast.  This is the value of
// attending fp32(code * scale + zero) up to fp32 rounding.
//
// Online softmax in the log2 domain; each warp writes one (m, l, o) partial per segment
// piece it covered; at the end each CTA merges its warps' partials per segment (one
// barrier), and the last CTA to finish a segment (an atomic arrival count, reset by that
// CTA) merges the CTA partials of the segment:
// M = max m_i, L = sum l_i 2^(m_i - M), o = sum o_i 2^(m_i - M) / L.
// Launched with programmatic stream serialization: the prologue up to griddepcontrol.wait
// overlaps the previous kernel's tail.
#include <math.h>

#include <atomic>

#include "kvq_internal.cuh"
#include "page_math.cuh"
#include "ptx.cuh"

namespace kvq {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
// Bytes of page staging per warp: three 16-bit pages at D = 128 with one CTA per SM (the
// 16-bit-only kernel, whose pages are bandwidth-bound); half that with two CTAs per SM (the
// kernel for caches with quantised pools, whose page math is latency-bound: twice the warps).
constexpr int kRingWide = 24576;
constexpr int kRingNarrow = 12288;
constexpr int kNBar = 8;      // pages in flight per warp (max)

struct PageMeta {
  int ring_off;  // byte offset of the K chunk in the warp ring
  int end;       // monotonic end of the allocation (ring bytes issued so far)
  int tier;      // -1: page skipped
  int nv;        // valid tokens
  int group;     // host-memory page: sequence number of its per-lane copy group, else -1
};

struct AttnArgs {
  DevCache c;
  const uint16_t* q;
  const int32_t* sel;
  const int32_t* cnt;
  int kmax;
  float scale_log2;
  float* wp_o;   // [wslots][G][D]  one partial per (worker warp, segment it touched)
  float* wp_ml;  // [wslots][G][2]
  float* ws_o;   // [slots][G][D]   one partial per (CTA, segment it touched)
  float* ws_ml;  // [slots][G][2]
  unsigned* counters;  // [B*Hkv] CTAs finished per segment (zero between calls)
  int num_ctas;
};

// Where one upcoming page lives; lane i of a warp holds the descriptor of the warp's
// i-th next page, so the dependent loads (page list -> block table) are paid once per
// 32 pages instead of once per page.
struct PageDesc {
  const unsigned char* src;   // K chunk
  const unsigned char* vsrc;  // V chunk (right after K unless the tier has a separate V pool)
  int tier;  // -1: skip
  int nv;
};

// Write the merged (M, L, o) of elements (h, d .. d+3) of segment bg: as a partial into
// slot `dst` of (dst_o, dst_ml), or, with dst < 0, as the segment's output o / L and lse.
template <bool BF16>
__device__ inline void put_merged4(const AttnArgs& a, uint16_t* out, float* lse, int bg, int h, int d, int D, float M,
                                   float Ls, float4 o, float* dst_o, float* dst_ml, int dst) {
  const DevCache& c = a.c;
  const int G = c.G;
  if (dst >= 0) {
    *reinterpret_cast<float4*>(&dst_o[((size_t)dst * G + h) * D + d]) = o;
    if (d == 0) *reinterpret_cast<float2*>(&dst_ml[((size_t)dst * G + h) * 2]) = make_float2(M, Ls);
    return;
  }
  const int b = bg / c.Hkv, g = bg % c.Hkv;
  const bool any = !(Ls <= 0.f);  // a NaN sum (a NaN key or value) gives a NaN output
  const float ov[4] = {o.x, o.y, o.z, o.w};
  const size_t oi = ((size_t)b * c.Hq + (size_t)g * G + h) * D + d;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float r = any ? ov[i] / Ls : 0.f;
    if constexpr (BF16) out[oi + i] = __bfloat16_as_ushort(__float2bfloat16_rn(r));
    else out[oi + i] = __half_as_ushort(__float2half_rn(r));
  }
  if (d == 0 && lse != nullptr)
    lse[(size_t)b * c.Hq + (size_t)g * G + h] = any ? (M + log2f(Ls)) * 0.69314718055994531f : -INFINITY;
}

// CTA merge of elements (h, d .. d+3) of segment bg: warps w0..w1 of this CTA hold one
// partial each, in their own ring (shared memory: the warp's last segment) or in their
// global warp slot (u + bg).  Every partial is loaded before any is used (one memory round
// trip).  The result goes to CTA partial slot `dst`, or to the output (dst < 0).
template <int D, bool BF16>
__device__ inline void cta_merge4(const AttnArgs& a, uint16_t* out, float* lse, const unsigned char* rings,
                                  int ring_bytes, const int* pseg, int bg, int h, int d, int w0, int w1, int dst) {
  const int G = a.c.G;
  float mv[kWarps], lv[kWarps];
  float4 ov[kWarps];
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    mv[w] = -INFINITY;
    lv[w] = 0.f;
    ov[w] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (w >= w0 && w <= w1) {
      if (pseg[w] == bg) {
        const float* sp = reinterpret_cast<const float*>(rings + (size_t)w * ring_bytes);
        ov[w] = *reinterpret_cast<const float4*>(&sp[h * D + d]);
        mv[w] = sp[G * D + 2 * h];
        lv[w] = sp[G * D + 2 * h + 1];
      } else {
        const size_t slot = (size_t)blockIdx.x * kWarps + w + bg;
        ov[w] = __ldcg(reinterpret_cast<const float4*>(&a.wp_o[(slot * G + h) * D + d]));
        const float2 ml = __ldcg(reinterpret_cast<const float2*>(&a.wp_ml[(slot * G + h) * 2]));
        mv[w] = ml.x;
        lv[w] = ml.y;
      }
    }
  }
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mv[w]);
  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
  float Ls = 0.f;
  if (M != -INFINITY) {
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float f = mv[w] == -INFINITY ? 0.f : exp2f(mv[w] - M);
      o.x += ov[w].x * f;
      o.y += ov[w].y * f;
      o.z += ov[w].z * f;
      o.w += ov[w].w * f;
      Ls += lv[w] * f;
    }
  }
  put_merged4<BF16>(a, out, lse, bg, h, d, D, M, Ls, o, a.ws_o, a.ws_ml, dst);
}

// Final merge of elements (h, d .. d+3) of segment bg from its CTA partial slots n0 + bg ..
// n1 + bg into the output; partials are read in batches of 8 with an online rescale (one
// round trip per batch).
template <int D, bool BF16>
__device__ inline void final_combine4(const AttnArgs& a, uint16_t* out, float* lse, int bg, int h, int d, int n0,
                                      int n1) {
  constexpr int NB = 8;
  const int G = a.c.G;
  float M = -INFINITY, Ls = 0.f;
  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j0 = n0; j0 <= n1; j0 += NB) {
    float mv[NB], lv[NB];
    float4 ov[NB];
#pragma unroll
    for (int i = 0; i < NB; ++i) {
      mv[i] = -INFINITY;
      lv[i] = 0.f;
      ov[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j0 + i <= n1) {
        const size_t slot = (size_t)(j0 + i) + bg;
        const float2 ml = __ldcg(reinterpret_cast<const float2*>(&a.ws_ml[(slot * G + h) * 2]));
        mv[i] = ml.x;
        lv[i] = ml.y;
        ov[i] = __ldcg(reinterpret_cast<const float4*>(&a.ws_o[(slot * G + h) * D + d]));
      }
    }
    float Mn = M;
#pragma unroll
    for (int i = 0; i < NB; ++i) Mn = fmaxf(Mn, mv[i]);
    if (Mn == -INFINITY) continue;
    const float r = M == -INFINITY ? 0.f : exp2f(M - Mn);
    o.x *= r;
    o.y *= r;
    o.z *= r;
    o.w *= r;
    Ls *= r;
#pragma unroll
    for (int i = 0; i < NB; ++i) {
      const float f = mv[i] == -INFINITY ? 0.f : exp2f(mv[i] - Mn);
      o.x += ov[i].x * f;
      o.y += ov[i].y * f;
      o.z += ov[i].z * f;
      o.w += ov[i].w * f;
      Ls += lv[i] * f;
    }
    M = Mn;
  }
  put_merged4<BF16>(a, out, lse, bg, h, d, D, M, Ls, o, nullptr, nullptr, -1);
}

template <int D, bool BF16, bool ONLY16, int kRing>
__global__ void __launch_bounds__(kThreads, kRing == kRingWide ? 1 : 2)
    attn_kernel(AttnArgs a, uint16_t* __restrict__ out, float* __restrict__ lse) {
  extern __shared__ __align__(128) unsigned char smem[];
  const DevCache& c = a.c;
  const int G = c.G;
  const int BH = c.B * c.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nworkers = a.num_ctas * kWarps;
  const int u = blockIdx.x * kWarps + warp;

  unsigned char* ring = smem + (size_t)warp * kRing;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)kWarps * kRing) + warp * kNBar;
  PageMeta* pmeta = reinterpret_cast<PageMeta*>(smem + (size_t)kWarps * kRing + kWarps * kNBar * 8) + warp * kNBar;
  int* off = reinterpret_cast<int*>(smem + (size_t)kWarps * kRing + kWarps * kNBar * 8 +
                                    kWarps * kNBar * sizeof(PageMeta));  // [BH + 1]
  int16_t* last_list = reinterpret_cast<int16_t*>(off + BH + 1);       // [BH] segments this CTA completes
  __shared__ int scan_sh[kWarps + 1];

  if (lane == 0) {
    for (int i = 0; i < kNBar; ++i) mbar_init(smem_u32(&bars[i]), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  fence_proxy_async();
  __syncwarp();

  // L2 prefetch of the block table and the queries, overlapping the previous kernel's
  // tail: the page lookups after the wait then hit L2 (a prefetch is only a hint; neither
  // array is written by the kernels this launch may overlap).
  {
    const size_t stride = (size_t)gridDim.x * kThreads * 128;
    const size_t nbt = (size_t)c.B * c.max_pages * sizeof(int32_t), nq = (size_t)c.B * c.Hq * D * 2;
    for (size_t o = ((size_t)blockIdx.x * kThreads + tid) * 128; o < nbt; o += stride)
      prefetch_l2_line(reinterpret_cast<const unsigned char*>(c.block_table) + o);
    for (size_t o = ((size_t)blockIdx.x * kThreads + tid) * 128; o < nq; o += stride)
      prefetch_l2_line(reinterpret_cast<const unsigned char*>(a.q) + o);
  }
  griddep_wait();  // the page lists and the cache come from earlier kernels
  const unsigned long long wait_ns = wait_limit_ns(a.counters, kWaitLimitWord);

  // segment offsets: exclusive prefix sum of the (clamped) selected counts
  {
    const int per = (BH + kThreads - 1) / kThreads;
    const int lo = min(BH, tid * per), hi = min(BH, lo + per);
    int s = 0;
    for (int i = lo; i < hi; ++i) s += min(max(a.cnt[i], 0), a.kmax);
    int x = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) scan_sh[warp] = x;
    __syncthreads();
    if (tid == 0) {
      int run = 0;
      for (int i = 0; i < kWarps; ++i) {
        const int t = scan_sh[i];
        scan_sh[i] = run;
        run += t;
      }
      scan_sh[kWarps] = run;
    }
    __syncthreads();
    int run = scan_sh[warp] + x - s;
    for (int i = lo; i < hi; ++i) {
      off[i] = run;
      run += min(max(a.cnt[i], 0), a.kmax);
    }
    if (tid == 0) off[BH] = scan_sh[kWarps];
    __syncthreads();
  }
  const int total = off[BH];
  const int W = (total + nworkers - 1) / nworkers;
  // segments with nothing selected: zero output, -inf lse (every nworkers-th segment here)
  for (int bg = u; bg < BH; bg += nworkers) {
    if (off[bg + 1] != off[bg]) continue;
    const int b = bg / c.Hkv, g = bg % c.Hkv;
    for (int e = lane; e < G * D; e += 32) {
      const int h = e / D, d = e % D;
      out[((size_t)b * c.Hq + (size_t)g * G + h) * D + d] = 0;
      if (d == 0 && lse != nullptr) lse[(size_t)b * c.Hq + (size_t)g * G + h] = -INFINITY;
    }
  }
  const int f0 = min(total, u * W);
  const int f1 = min(total, f0 + W);

  int issued = 0, consumed = 0;  // pages of [f0, f1) issued / consumed
  int groups = 0;                // per-lane copy groups committed (host-memory pages)
  int head = 0, tail = 0;        // monotonic ring byte counters
  int win_base = 0, win_n = 0;   // descriptor window: pages [f0 + win_base, f0 + win_base + win_n)
  PageDesc my{nullptr, nullptr, -1, 0};
  bool failed = false;
  const unsigned char* ring_c = ring;

  // lane i: descriptor of page f0 + issued + i (binary search of its segment in off[])
  int my_rank = lane;  // issue position of this lane's page within the window
  auto prefetch = [&]() {
    win_base = issued;
    win_n = min(32, (f1 - f0) - issued);
    int bgw = 0;  // segment of this lane's page
    my = PageDesc{nullptr, nullptr, -1, 0};
    if (lane < win_n) {
      const int f = f0 + issued + lane;
      int lo = 0, hi = BH - 1;  // last bg with off[bg] <= f
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (off[mid] <= f) lo = mid; else hi = mid - 1;
      }
      const int bg = lo;
      bgw = bg;
      const int b = bg / c.Hkv, g = bg % c.Hkv;
      const int p = __ldg(&a.sel[(size_t)bg * a.kmax + (f - off[bg])]);
      const int L = __ldg(&c.seq_len[b]);
      const int P = min((L + kPage - 1) / kPage, c.max_pages);
      if (p >= 0 && p < P) {
        int tier;
        const unsigned char *src, *vsrc;
        if (page_chunks(c, b, p, g, tier, src, vsrc)) {
          my.src = src;
          my.vsrc = vsrc;
          my.tier = tier;
          my.nv = min(kPage, L - p * kPage);
        }
      } else {
        set_err(c.err, KVQ_DERR_BAD_PAGE);
      }
    }
    if constexpr (!ONLY16) {
      // Issue the window's pages grouped by tier inside each segment (segments stay in
      // order, so the k-th page issued is still in the segment of the k-th flat page):
      // a warp then runs one tier's page math at a time, which keeps the instruction cache
      // from cycling through every tier's code.  rank = position in (segment, tier, lane)
      // order; the page issued k-th is the lane whose rank is k.
      // Segments are contiguous in lane order (lanes past the window form a group of their
      // own after them), so rank = lanes of earlier segments + lanes of this segment with a
      // lower tier + lanes of this segment and tier before this one.
      const int seg = lane < win_n ? bgw : 0x7FFFFFFF;
      const int tier_k = lane < win_n && my.tier >= 0 ? my.tier : 7;
      const unsigned same_seg = __match_any_sync(0xffffffffu, seg);
      unsigned lower = 0u, same_tier = 0u;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const unsigned m = __ballot_sync(0xffffffffu, tier_k == t);
        if (t < tier_k) lower |= m;
        if (t == tier_k) same_tier = m;
      }
      const unsigned before = (1u << lane) - 1u;
      my_rank = (__ffs(same_seg) - 1) + __popc(lower & same_seg) + __popc(same_tier & same_seg & before);
    }
  };

  auto issue_more = [&]() {
    while (issued - consumed < kNBar && issued < f1 - f0) {
      if (issued == win_base + win_n) prefetch();
      const int k = ONLY16 ? issued - win_base
                           : __ffs(__ballot_sync(0xffffffffu, my_rank == issued - win_base)) - 1;
      const unsigned long long sp = __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(my.src), k);
      const unsigned long long vp = __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(my.vsrc), k);
      const int tier = __shfl_sync(0xffffffffu, my.tier, k);
      const int nv = __shfl_sync(0xffffffffu, my.nv, k);
      const int cb = tier >= 0 ? c.chunk[tier] : 0;
      const int bytes = 2 * cb;
      // An empty ring (every issued page consumed) restarts at offset 0, so a page of up to
      // kRing bytes always fits; otherwise the page goes after the last one issued, or to
      // the ring's start when it does not fit before the end, once that space is consumed.
      if (issued == consumed) head = tail = 0;
      int start = head;
      const int pos = head % kRing;
      if (pos + bytes > kRing) start += kRing - pos;
      if (start + bytes - tail > kRing) break;  // no room yet
      const int slot = issued % kNBar;
      const uint32_t bar = smem_u32(&bars[slot]);
      // K and V chunks of a pool in pinned host memory are fetched by every lane with
      // 16-byte asynchronous loads (one commit group per page); device chunks by bulk copy
      const bool khost = bytes > 0 && ((c.host_tiers >> tier) & 1u);
      const bool vhost = bytes > 0 && (c.vpool[tier] != nullptr ? ((c.host_vtiers >> tier) & 1u) != 0u : khost);
      const bool host = khost || vhost;
      const uint32_t dst = smem_u32(ring + start % kRing);
      if (host) {
        const unsigned char* ks = reinterpret_cast<const unsigned char*>(sp);
        const unsigned char* vs = reinterpret_cast<const unsigned char*>(vp);
        if (khost)
          for (int o = lane * 16; o < cb; o += 32 * 16) cp_async16(dst + o, ks + o);
        if (vhost)
          for (int o = lane * 16; o < cb; o += 32 * 16) cp_async16(dst + cb + o, vs + o);
        cp_async_commit();
      }
      if (lane == 0) {
        pmeta[slot] = PageMeta{start % kRing, start + bytes, tier, nv, host ? groups : -1};
        const uint32_t tx = (khost ? 0u : (uint32_t)cb) + (vhost ? 0u : (uint32_t)cb);
        if (bytes > 0 && tx > 0) {
          mbar_expect_tx(bar, tx);
          if (!host && vp == sp + (unsigned long long)cb) {  // adjacent K and V: one copy
            bulk_copy_g2s(dst, reinterpret_cast<const void*>(sp), (uint32_t)bytes, bar);
          } else {
            if (!khost) bulk_copy_g2s(dst, reinterpret_cast<const void*>(sp), (uint32_t)cb, bar);
            if (!vhost) bulk_copy_g2s(dst + cb, reinterpret_cast<const void*>(vp), (uint32_t)cb, bar);
          }
        } else {
          mbar_arrive(bar);
        }
      }
      groups += host ? 1 : 0;
      head = start + bytes;
      ++issued;
    }
    __syncwarp();
  };

  issue_more();  // start the copies before anything else

  WarpState<D> st;
  int cur = -1;  // segment being accumulated
  int bg = 0;    // segment of page f0 + k: pages are contiguous, so a forward cursor suffices
  {
    int lo = 0, hi = BH - 1;  // last segment starting at or before f0
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (off[mid] <= f0) lo = mid; else hi = mid - 1;
    }
    bg = lo;
  }
  for (int k = 0; k < f1 - f0; ++k) {
    if (!failed) issue_more();
    const int slot = consumed % kNBar;
    const uint32_t parity = (consumed / kNBar) & 1;
    while (off[bg + 1] <= f0 + k) ++bg;  // skip finished and empty segments
    if (bg != cur) {
      if (cur >= 0) write_warp_partial<D>(G, st, a.wp_o + (size_t)(u + cur) * G * D, a.wp_ml + (size_t)(u + cur) * G * 2, lane);
      cur = bg;
      begin_segment<D, BF16>(a.q, c.Hq, G, bg / c.Hkv, bg % c.Hkv, lane, st);
    }
    if (!failed) {
      const bool ok = mbar_wait_bounded(smem_u32(&bars[slot]), parity, wait_ns);
      if (__any_sync(0xffffffffu, !ok)) {
        failed = true;
        if (lane == 0) set_err(c.err, KVQ_DERR_TIMEOUT);
      }
    }
    if (!failed) {
      const PageMeta pm = pmeta[slot];
      if (pm.group >= 0) {  // wait for this page's group (later pages' groups may stay in flight)
        cp_async_wait_pending(groups - 1 - pm.group);
        __syncwarp();
      }
      if (pm.tier >= 0) process_page<D, BF16, ONLY16>(ring_c + pm.ring_off, pm.tier, pm.nv, lane, a.scale_log2, st);
      if (pm.group >= 0) fence_proxy_async();  // generic-proxy writes, before a bulk copy may reuse the bytes
      tail = pm.end;  // everything before this page's end is free again
    }
    __syncwarp();
    ++consumed;
  }
  // the last segment's partial goes to this warp's ring (every copy has been consumed),
  // earlier ones went to the warp's global slots
  __shared__ int s_pseg[kWarps];
  if (cur >= 0 && !failed) {
    float* sp = reinterpret_cast<float*>(ring);
    write_warp_partial<D>(G, st, sp, sp + G * D, lane);
  } else if (cur >= 0) {
    write_warp_partial<D>(G, st, a.wp_o + (size_t)(u + cur) * G * D, a.wp_ml + (size_t)(u + cur) * G * 2, lane);
  }
  if (lane == 0) s_pseg[warp] = failed ? -1 : cur;
  // after a timeout, give copies still in flight a bounded chance to land before exit
  if (failed) {
    for (int k = consumed; k < issued; ++k) mbar_wait_bounded(smem_u32(&bars[k % kNBar]), (k / kNBar) & 1, wait_ns);
  }
  if (groups > 0) cp_async_wait_pending(0);  // no per-lane copy may land after this point

  // Merge, in three phases over all the segments this CTA touched at once (a CTA-wide
  // barrier between phases, so the tail costs a few memory round trips however many
  // segments the CTA holds):
  //  1. per (segment, element): merge this CTA's warp partials; a segment that lies inside
  //     the CTA goes straight to the output, others to the CTA's partial slot;
  //  2. per segment spanning CTAs: count this CTA's arrival; the last CTA to arrive
  //     (no waiting) resets the counter and lists the segment;
  //  3. per (listed segment, element): merge the segment's CTA partials into the output.
  __syncthreads();
  const int cw = kWarps * W;  // pages per CTA
  const int cta0 = min(total, (int)blockIdx.x * cw), cta1 = min(total, cta0 + cw);
  __shared__ int s_nlast;
  if (cta0 < cta1) {
    auto seg_of = [&](int f) {  // last segment starting at or before flat page f
      int lo = 0, hi = BH - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (off[mid] <= f) lo = mid; else hi = mid - 1;
      }
      return lo;
    };
    const int s0 = seg_of(cta0), s1 = seg_of(cta1 - 1);
    const int nseg = s1 - s0 + 1, GD = G * D / 4;  // units of 4 consecutive channels
    const int wb = (int)blockIdx.x * kWarps;
    for (int e = tid; e < nseg * GD; e += kThreads) {
      const int sbg = s0 + e / GD, el = e % GD;
      if (off[sbg + 1] == off[sbg]) continue;  // empty segment: written at the start
      const int w0 = max(wb, off[sbg] / W) - wb;
      const int w1 = min(wb + kWarps - 1, (off[sbg + 1] - 1) / W) - wb;
      const int n0 = off[sbg] / cw, n1 = (off[sbg + 1] - 1) / cw;
      cta_merge4<D, BF16>(a, out, lse, smem, kRing, s_pseg, sbg, el / (D / 4), 4 * (el % (D / 4)), w0, w1,
                          n0 == n1 ? -1 : (int)blockIdx.x + sbg);
    }
    __threadfence();  // this thread's CTA partials are visible before any arrival is counted
    if (tid == 0) s_nlast = 0;
    __syncthreads();
    for (int i = tid; i < nseg; i += kThreads) {
      const int sbg = s0 + i;
      if (off[sbg + 1] == off[sbg]) continue;
      const int n0 = off[sbg] / cw, n1 = (off[sbg + 1] - 1) / cw;
      if (n0 == n1) continue;  // the whole segment was in this CTA: output written
      const unsigned old = atomicAdd(&a.counters[sbg], 1u);
      if (old == static_cast<unsigned>(n1 - n0)) {  // every CTA of the segment has arrived
        a.counters[sbg] = 0u;                          // ready for the next call
        last_list[atomicAdd(&s_nlast, 1)] = static_cast<int16_t>(sbg);
      }
    }
    __syncthreads();
    const int nl = s_nlast;
    if (nl > 0) {
      __threadfence();
      for (int e = tid; e < nl * GD; e += kThreads) {
        const int sbg = last_list[e / GD], el = e % GD;
        const int n0 = off[sbg] / cw, n1 = (off[sbg + 1] - 1) / cw;
        final_combine4<D, BF16>(a, out, lse, sbg, el / (D / 4), 4 * (el % (D / 4)), n0, n1);
      }
    }
  }
  griddep_launch_dependents();
}

// Dynamic shared memory: the warps' rings, their mbarriers and page records, then the
// segment offsets [BH + 1] and the list of segments a CTA completes [BH] (int16).
size_t attn_smem_bytes(int ring, int BH) {
  return (size_t)kWarps * ring + kWarps * kNBar * 8 + kWarps * kNBar * sizeof(PageMeta) + (size_t)(BH + 1) * 4 +
         ((size_t)BH * 2 + 15) / 16 * 16;
}

bool only16_cache(const DevCache& c) {
  for (int t = 1; t < kNumTiers; ++t)
    if (c.pool[t] != nullptr) return false;
  return true;
}

// Two CTAs per SM when the cache has quantised pools and two narrow-ring CTAs fit (228 KB
// of shared memory per SM, 1 KB of it reserved per CTA); one otherwise.
int ctas_per_sm(const DevCache& c) {
  if (only16_cache(c)) return 1;
  return 2 * (attn_smem_bytes(kRingNarrow, c.B * c.Hkv) + 1024) <= 233472 ? 2 : 1;
}

template <int D, bool BF16, bool ONLY16, int RING>
cudaError_t launch_attn_v(const AttnArgs& a, uint16_t* out, float* lse, cudaStream_t s) {
  const size_t smem = attn_smem_bytes(RING, a.c.B * a.c.Hkv);
  cudaError_t e = cudaFuncSetAttribute(attn_kernel<D, BF16, ONLY16, RING>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(attn_kernel<D, BF16, ONLY16, RING>, dim3(a.num_ctas), dim3(kThreads), smem, s, a, out, lse);
}

// A cache whose only pool is the 16-bit one runs the 16-bit-only kernel (one CTA per SM);
// others the all-tier kernel, two CTAs per SM when they fit.
template <int D, bool BF16>
cudaError_t launch_attn_d(const AttnArgs& a, uint16_t* out, float* lse, cudaStream_t s) {
  if (only16_cache(a.c)) return launch_attn_v<D, BF16, true, kRingWide>(a, out, lse, s);
  return ctas_per_sm(a.c) == 2 ? launch_attn_v<D, BF16, false, kRingNarrow>(a, out, lse, s)
                               : launch_attn_v<D, BF16, false, kRingWide>(a, out, lse, s);
}

}  // namespace

int sm_count(int device) {
  static int cache[64] = {0};
  if (device >= 0 && device < 64 && cache[device] > 0) return cache[device];
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || sms <= 0) sms = 148;
  if (device >= 0 && device < 64) cache[device] = sms;
  return sms;
}

namespace {
std::atomic<int> g_grid_override{0};
}

void set_grid_override(int ctas) { g_grid_override.store(ctas > 0 ? ctas : 0); }

int attn_num_ctas(int device) {
  const int o = g_grid_override.load();
  return o > 0 ? o : sm_count(device);
}

int attn_grid(const DevCache& c, int device) {
  const int o = g_grid_override.load();
  return o > 0 ? o : sm_count(device) * ctas_per_sm(c);
}

// Workspace: [kCounterBytes] per-segment arrival counters (zero between calls, at a fixed
// place so that any later call, whatever its shapes, finds them zero), then the o parts of
// the warp partials ([wslots][G][D]; wslots = warps + B*Hkv) and of the CTA partials
// ([slots][G][D]; slots = CTAs + B*Hkv), then their (m, l) parts ([wslots][G][2],
// [slots][G][2]).  A warp (CTA) u that
// covers segment bg writes slot u + bg: unique because ranges are contiguous and ordered.
size_t attn_workspace_bytes(const DevCache& c, int num_ctas) {
  const size_t BH = (size_t)c.B * c.Hkv;
  const size_t wslots = (size_t)num_ctas * kWarps + BH, slots = (size_t)num_ctas + BH;
  return kCounterBytes + (wslots + slots) * c.G * ((size_t)c.D + 2) * sizeof(float);
}

cudaError_t launch_attn(const DevCache& c, const void* q, const int32_t* sel, const int32_t* cnt, int kmax,
                        float sm_scale, void* out, float* lse, void* ws, int num_ctas, cudaStream_t s) {
  AttnArgs a;
  a.c = c;
  a.q = static_cast<const uint16_t*>(q);
  a.sel = sel;
  a.cnt = cnt;
  a.kmax = kmax;
  a.scale_log2 = sm_scale * 1.4426950408889634f;
  const size_t BH = (size_t)c.B * c.Hkv;
  const size_t wslots = (size_t)num_ctas * kWarps + BH, slots = (size_t)num_ctas + BH;
  a.counters = static_cast<unsigned*>(ws);
  a.wp_o = reinterpret_cast<float*>(static_cast<unsigned char*>(ws) + kCounterBytes);
  a.ws_o = a.wp_o + wslots * c.G * c.D;  // o arrays first: every row 16-byte aligned
  a.wp_ml = a.ws_o + slots * c.G * c.D;
  a.ws_ml = a.wp_ml + wslots * c.G * 2;
  a.num_ctas = num_ctas;
  uint16_t* o = static_cast<uint16_t*>(out);
  const bool bf = c.dtype == KVQ_DT_BF16;
  if (c.D == 128) return bf ? launch_attn_d<128, true>(a, o, lse, s) : launch_attn_d<128, false>(a, o, lse, s);
  if (c.D == 64) return bf ? launch_attn_d<64, true>(a, o, lse, s) : launch_attn_d<64, false>(a, o, lse, s);
  return cudaErrorInvalidValue;
}

}  // namespace kvq
