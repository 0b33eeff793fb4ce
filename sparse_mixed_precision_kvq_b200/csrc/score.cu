// kvq_page_scores: page score from the mean-key summary.
//
// AMASS "decode-time sparse KV-cache attention for vLLM", "What is in the box": pages are
// ranked by a compact score computed from a tiny resident per-page summary; the score
// kernel is a bandwidth-bound sweep over all summaries.  Score of page p for kv head g:
//   s[b][g][p] = max_{h in group g} sum_d q[b][h][d] * kbar[b][g][p][d]
//
// The sweep runs on the tensor core, one warp per 16-page tile (score_tile.cuh); each
// lane reads its share of the summary rows straight from global memory with 16-byte
// loads, double-buffered in registers.
#include <math.h>

#include "kvq_internal.cuh"
#include "quant.cuh"
#include "score_tile.cuh"
#include "select_core.cuh"
#include "tile_split.cuh"

namespace kvq {
namespace {

constexpr int kScoreWarps = 8;

template <int D>
__device__ inline void load_tile(const uint16_t* sbase, int tile, int P, int lane, uint4 (&av)[2][D / 32]) {
  constexpr int CW = D / 4;
  const int g8 = lane >> 2, q4 = lane & 3;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int p = tile * 16 + g8 + 8 * r;
    const uint4* src = reinterpret_cast<const uint4*>(sbase + (size_t)p * D + CW * q4);
#pragma unroll
    for (int i = 0; i < CW / 8; ++i) av[r][i] = p < P ? __ldcg(src + i) : make_uint4(0, 0, 0, 0);
  }
}

// Extra work of the fused form (kvq_score_select): the token append before the scores
// and the selection after them.
struct ScoreSelect {
  const int32_t* pos;  // nullable: no append
  const uint16_t* k_new;
  const uint16_t* v_new;
  kvq_select_params prm;
  int32_t* sel;
  int32_t* cnt;
  int kmax;
  unsigned* done;  // [B * Hkv] tiles scored per (b, g) (zero between calls)
};

// Grid of 2 CTAs per SM; warp w takes a contiguous run of the flat list of 16-page tiles
// in (b, g, tile) order (which tiles the list holds: REAL below), loading the next tile
// while the current one is multiplied.
// MODE 1 (kvq_append_scores): the append kernel runs just before this one and writes
// only the summary row of page pos[b] / 16 of each (b, g).  Every other tile is scored
// before waiting for that kernel, so the sweep overlaps the append; the tiles holding an
// appended page are scored after the wait.
// MODE 2 (kvq_score_select): the warp that owns the tile of a (b, g)'s appended token
// writes the token first (so that tile is read after the new summary row is stored);
// after its tiles, the CTA counts them on each (b, g) it touched, and the CTA that
// completes a (b, g) selects its pages (select_core.cuh) from the scores in L2.
enum { SCORES = 0, APPEND_SCORES = 1, APPEND_SCORES_SELECT = 2 };

// REAL (modes 0 and 1): only the tiles that hold pages are divided among the warps
// (tile_split.cuh); otherwise every row's max_pages / 16 tiles.
template <int D, bool BF16, int MODE, bool REAL>
__global__ void __launch_bounds__(kScoreWarps * 32, 2) score_kernel(DevCache c, const uint16_t* __restrict__ q,
                                                                    float* __restrict__ scores, int tiles_per_bg,
                                                                    int per, ScoreSelect f) {
  // MODE 2: keys [max_pages], then the selection scratch; REAL: the tile prefix [B * Hkv + 1]
  extern __shared__ __align__(16) uint32_t sel_smem[];
  __shared__ SelShared sel_sh;
  __shared__ int s_unit;
  __shared__ int s_part[kScoreWarps];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, q4 = lane & 3;
  const int BH = c.B * c.Hkv;
  const int nw = gridDim.x * kScoreWarps, gw = blockIdx.x * kScoreWarps + warp;
  int* pre = reinterpret_cast<int*>(sel_smem);
  // Reads before the wait go to L2 (__ldcg): what they touch was written by grids that are
  // complete, and no stale L1 line may stand in for it.
  auto pages_of = [&](int bg) { return row_pages(c, bg); };
  int total, i0, i1;
  if constexpr (REAL) {
    total = row_tile_prefix<kScoreWarps * 32>(c, pre, s_part, tid);
    const int pw = (total + nw - 1) / nw;
    i0 = min(total, gw * pw);
    i1 = min(total, i0 + pw);
  } else {
    total = BH * tiles_per_bg;
    i0 = gw * per;
    i1 = min(total, i0 + per);
  }
  // (b, g) of item i
  auto bg_at = [&](int i) {
    if constexpr (REAL) return row_of_item(pre, BH, i);
    else return i / tiles_per_bg;
  };
  // the same with a forward cursor (items visited in increasing order), and the tile
  auto locate = [&](int i, int& cur, int& tile) {
    if constexpr (REAL) {
      advance_row(pre, cur, i);
      tile = i - pre[cur];
      return cur;
    } else {
      tile = i % tiles_per_bg;
      return i / tiles_per_bg;
    }
  };
  // Before waiting for the previous kernel (the append, which writes only the open page's
  // summary row): ask L2 for this warp's summary rows, one bulk prefetch per (b, g) piece,
  // so their DRAM traffic overlaps that kernel (a prefetch is only a hint).  MODE 1 reads
  // them at once instead (measured faster than a prefetch ahead of the sweep).
  if (MODE != APPEND_SCORES && lane == 0 && i0 < i1) {
    int cur = bg_at(i0);
    for (int i = i0; i < i1;) {
      int tile;
      const int bg = locate(i, cur, tile);
      const int n = min(i1, REAL ? pre[bg + 1] : (bg + 1) * tiles_per_bg) - i;  // tiles of this piece
      const int p0 = tile * 16, p1 = min(pages_of(bg), (tile + n) * 16);
      if (p1 > p0) bulk_prefetch_l2(c.summary + ((size_t)bg * c.max_pages + p0) * D, (uint32_t)(p1 - p0) * D * 2);
      i += n;
    }
  }
  if constexpr (MODE != APPEND_SCORES) griddep_wait();

  if (MODE == APPEND_SCORES_SELECT && f.pos != nullptr && i0 < i1) {  // appends whose page lies in this warp's tiles
    for (int bg = i0 / tiles_per_bg; bg <= (i1 - 1) / tiles_per_bg; ++bg) {
      const int b = bg / c.Hkv, g = bg % c.Hkv;
      const int ps = f.pos[b];
      if (ps < 0) continue;
      if (ps >= c.max_pages * kPage) {
        if (lane == 0 && g == 0 && bg * tiles_per_bg >= i0) set_err(c.err, KVQ_DERR_BAD_POS);
        continue;
      }
      const int it = bg * tiles_per_bg + (ps / kPage) / 16;
      if (it < i0 || it >= i1) continue;
      append_token_warp<BF16>(c, b, g, ps, f.k_new + (size_t)bg * D, f.v_new + (size_t)bg * D, lane, nullptr);
      __syncwarp();
    }
  }
  if constexpr (REAL) fill_past_tiles(c, pre, scores, gw, nw, lane);

  if (i0 < i1) {
    QFrag<D, BF16> qf;
    int cur_bg = -1, P = 0;
    float* out = nullptr;
    bool bad = false;
    uint4 av0[2][D / 32], av1[2][D / 32];  // double buffer (compile-time indexed)
    int lcur = bg_at(i0), ccur = lcur;      // cursors of the loads and of the math

    auto tile_src = [&](int i, int& Pn, int& tile) -> const uint16_t* {
      const int bg = locate(i, lcur, tile);
      Pn = pages_of(bg);
      return c.summary + (size_t)bg * c.max_pages * D;
    };
    auto compute = [&](int i, const uint4 (&av)[2][D / 32]) {
      int tile;
      const int bg = locate(i, ccur, tile);
      if (bg != cur_bg) {  // new (b, g): its query fragments (hi + lo)
        cur_bg = bg;
        const int b = bg / c.Hkv, g = bg % c.Hkv;
        P = pages_of(bg);
        out = scores + (size_t)bg * c.max_pages;
        qf.load(q, c.Hq, c.G, b, g, lane, bad);
      }
      float m0, m1;
      tile_scores<D, BF16>(av, qf, c.G, lane, m0, m1);
      if (q4 == 0) {
        const int p0 = tile * 16 + g8, p1 = p0 + 8;
        if (p0 < c.max_pages) out[p0] = p0 < P ? m0 : -INFINITY;
        if (p1 < c.max_pages) out[p1] = p1 < P ? m1 : -INFINITY;
      }
    };
    auto load = [&](int i, uint4 (&av)[2][D / 32]) {
      int Pn, tile;
      const uint16_t* src = tile_src(i, Pn, tile);
      load_tile<D>(src, tile, Pn, lane, av);
    };

    // MODE 1: the item holding the appended page of each (b, g) in this warp's run; lane j
    // keeps that of (b, g) bg0 + j (-1: none).  pos is the caller's, not the append's.
    const int bg0 = bg_at(i0), bg1 = bg_at(i1 - 1);
    auto aff_of = [&](int bg) {
      const int ps = __ldcg(&f.pos[bg / c.Hkv]);
      if (ps < 0 || ps >= c.max_pages * kPage) return -1;
      const int t = (ps / kPage) / 16;
      if constexpr (REAL) return t < pre[bg + 1] - pre[bg] ? pre[bg] + t : -1;
      else return bg * tiles_per_bg + t;
    };
    int my_aff = -1;
    if (MODE == APPEND_SCORES && bg0 + lane <= bg1) my_aff = aff_of(bg0 + lane);
    auto held_back = [&](int i) {  // uniform over the warp
      if constexpr (MODE != APPEND_SCORES) {
        return false;
      } else {
        if (bg1 - bg0 < 32) return __any_sync(0xffffffffu, my_aff == i) != 0;
        return aff_of(bg_at(i)) == i;
      }
    };
    auto next_tile = [&](int i) {  // the next tile after i scored before the wait
      for (++i; i < i1; ++i)
        if (!held_back(i)) break;
      return i;
    };
    if constexpr (MODE != APPEND_SCORES) {  // every tile of the run
      load(i0, av0);
      for (int i = i0; i < i1; i += 2) {
        if (i + 1 < i1) load(i + 1, av1);
        compute(i, av0);
        if (i + 1 >= i1) break;
        if (i + 2 < i1) load(i + 2, av0);
        compute(i + 1, av1);
      }
    }
    int i = MODE == APPEND_SCORES ? next_tile(i0 - 1) : i1;
    if (i < i1) {
      load(i, av0);
      while (true) {  // next tile into the odd buffer, then the even tile's math
        const int j = next_tile(i);
        if (j < i1) load(j, av1);
        compute(i, av0);
        if (j >= i1) break;
        const int k = next_tile(j);
        if (k < i1) load(k, av0);
        compute(j, av1);
        if (k >= i1) break;
        i = k;
      }
    }
    if constexpr (MODE == APPEND_SCORES) {
      griddep_wait();  // the appended tokens' summary rows are written (and this grid ends after the append)
      lcur = ccur = bg0;
      for (int t = i0; t < i1; ++t) {
        if (!held_back(t)) continue;
        load(t, av0);
        compute(t, av0);
      }
    }
    if (bad) set_err(c.err, KVQ_DERR_FP16_RANGE);
  }

  if constexpr (MODE == APPEND_SCORES_SELECT) {
    // count this CTA's tiles on each (b, g) it touched; the CTA completing one selects it
    const int c0 = min(total, (int)blockIdx.x * kScoreWarps * per);
    const int c1 = min(total, c0 + kScoreWarps * per);
    __syncthreads();
    if (c0 < c1) {
      for (int bg = c0 / tiles_per_bg; bg <= (c1 - 1) / tiles_per_bg; ++bg) {
        if (tid == 0) {  // the barrier orders every warp's score writes before this fence
          const int n = min(c1, (bg + 1) * tiles_per_bg) - max(c0, bg * tiles_per_bg);
          __threadfence();
          const unsigned old = atomicAdd(&f.done[bg], static_cast<unsigned>(n));
          s_unit = (old + static_cast<unsigned>(n) == static_cast<unsigned>(tiles_per_bg)) ? bg : -1;
          if (s_unit >= 0) f.done[bg] = 0u;  // complete: free for the next call
        }
        __syncthreads();
        if (s_unit == bg) {
          __threadfence();
          const int L = c.seq_len[bg / c.Hkv];
          const int P = min((L + kPage - 1) / kPage, c.max_pages);
          const float* sc = scores + (size_t)bg * c.max_pages;
          uint32_t* keys = sel_smem;
          bool nan_seen = false;
          for (int p0 = tid; p0 < P; p0 += 4 * kScoreWarps * 32) {  // four loads in flight per thread
            float v[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int p = p0 + j * kScoreWarps * 32;
              v[j] = p < P ? __ldcg(sc + p) : 0.f;
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int p = p0 + j * kScoreWarps * 32;
              if (p < P) keys[p] = order_key(v[j], nan_seen);
            }
          }
          if (nan_seen) set_err(c.err, KVQ_DERR_NAN_SCORE);
          __syncthreads();
          struct SyncBar {
            __device__ bool operator()() const {
              __syncthreads();
              return true;
            }
          } bar;
          select_pages<kScoreWarps * 32>(keys, P, f.prm, f.sel + (size_t)bg * f.kmax, f.cnt + bg, f.kmax, c.err,
                                         sel_smem + (c.max_pages + 3) / 4 * 4, sel_sh, tid, bar);
        }
        __syncthreads();
      }
    }
  }
  griddep_launch_dependents();
}

template <int D, bool BF16, int MODE>
cudaError_t launch_d(const DevCache& c, const void* q, float* scores, const ScoreSelect& f, cudaStream_t s) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  const int tiles_per_bg = (c.max_pages + 15) / 16;
  const long long total = (long long)c.B * c.Hkv * tiles_per_bg;  // every row full: the most tiles
  const long long blocks_max = 2LL * sm_count(dev);
  const long long warps = blocks_max * kScoreWarps;
  const int per = (int)((total + warps - 1) / warps);
  const long long blocks = (total + (long long)per * kScoreWarps - 1) / ((long long)per * kScoreWarps);
  if constexpr (MODE == APPEND_SCORES_SELECT) {
    const size_t smem = ((size_t)(c.max_pages + 3) / 4 * 4 + kSelScratchWords) * sizeof(uint32_t);
    const cudaError_t e = cudaFuncSetAttribute(score_kernel<D, BF16, MODE, false>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(score_kernel<D, BF16, MODE, false>, dim3((unsigned)blocks), dim3(kScoreWarps * 32), smem, s,
                      c, static_cast<const uint16_t*>(q), scores, tiles_per_bg, per, f);
  } else {
    // the tile prefix in shared memory while it fits the default 48 KB; whole rows beyond
    const size_t smem = ((size_t)c.B * c.Hkv + 1) * sizeof(int);
    if (smem <= 48 * 1024)
      return launch_pdl(score_kernel<D, BF16, MODE, true>, dim3((unsigned)blocks), dim3(kScoreWarps * 32), smem, s,
                        c, static_cast<const uint16_t*>(q), scores, tiles_per_bg, per, f);
    return launch_pdl(score_kernel<D, BF16, MODE, false>, dim3((unsigned)blocks), dim3(kScoreWarps * 32), 0, s, c,
                      static_cast<const uint16_t*>(q), scores, tiles_per_bg, per, f);
  }
}

}  // namespace

cudaError_t launch_scores(const DevCache& c, const void* q, float* scores, cudaStream_t s) {
  if (c.G > kMaxG) return cudaErrorInvalidValue;
  const bool bf = c.dtype == KVQ_DT_BF16;
  const ScoreSelect f{};
  if (c.D == 128) return bf ? launch_d<128, true, SCORES>(c, q, scores, f, s) : launch_d<128, false, SCORES>(c, q, scores, f, s);
  if (c.D == 64) return bf ? launch_d<64, true, SCORES>(c, q, scores, f, s) : launch_d<64, false, SCORES>(c, q, scores, f, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_score_select(const DevCache& c, const int32_t* pos, const void* k_new, const void* v_new,
                                const void* q, const kvq_select_params& prm, float* scores, int32_t* sel,
                                int32_t* cnt, int kmax, unsigned* done, cudaStream_t s) {
  if (c.G > kMaxG) return cudaErrorInvalidValue;
  const bool bf = c.dtype == KVQ_DT_BF16;
  const ScoreSelect f{pos, static_cast<const uint16_t*>(k_new), static_cast<const uint16_t*>(v_new), prm, sel, cnt,
                      kmax, done};
  if (c.D == 128)
    return bf ? launch_d<128, true, APPEND_SCORES_SELECT>(c, q, scores, f, s)
              : launch_d<128, false, APPEND_SCORES_SELECT>(c, q, scores, f, s);
  if (c.D == 64)
    return bf ? launch_d<64, true, APPEND_SCORES_SELECT>(c, q, scores, f, s)
              : launch_d<64, false, APPEND_SCORES_SELECT>(c, q, scores, f, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_append_scores(const DevCache& c, const int32_t* pos, const void* k_new, const void* v_new,
                                 const void* q, float* scores, cudaStream_t s) {
  if (c.G > kMaxG) return cudaErrorInvalidValue;
  const cudaError_t e = launch_append(c, pos, k_new, v_new, s);
  if (e != cudaSuccess) return e;
  const bool bf = c.dtype == KVQ_DT_BF16;
  ScoreSelect f{};
  f.pos = pos;
  f.k_new = static_cast<const uint16_t*>(k_new);
  f.v_new = static_cast<const uint16_t*>(v_new);
  if (c.D == 128)
    return bf ? launch_d<128, true, APPEND_SCORES>(c, q, scores, f, s) : launch_d<128, false, APPEND_SCORES>(c, q, scores, f, s);
  if (c.D == 64)
    return bf ? launch_d<64, true, APPEND_SCORES>(c, q, scores, f, s) : launch_d<64, false, APPEND_SCORES>(c, q, scores, f, s);
  return cudaErrorInvalidValue;
}

}  // namespace kvq
