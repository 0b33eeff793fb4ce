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
#include "score_tile.cuh"

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
    for (int i = 0; i < CW / 8; ++i) av[r][i] = p < P ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
  }
}

// Grid of 2 CTAs per SM; warp w takes the contiguous run of 16-page tiles
// [w * per, (w + 1) * per) of the flat list (b, g, tile), loading the next tile while
// the current one is multiplied.
template <int D, bool BF16>
__global__ void __launch_bounds__(kScoreWarps * 32, 2) score_kernel(DevCache c, const uint16_t* __restrict__ q,
                                                                    float* __restrict__ scores, int tiles_per_bg,
                                                                    int per) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g8 = lane >> 2, q4 = lane & 3;
  const int total = c.B * c.Hkv * tiles_per_bg;
  const int i0 = (blockIdx.x * kScoreWarps + warp) * per;
  const int i1 = min(total, i0 + per);
  griddep_wait();
  if (i0 >= i1) return;

  QFrag<D, BF16> qf;
  int cur_bg = -1, P = 0;
  float* out = nullptr;
  bool bad = false;
  uint4 av0[2][D / 32], av1[2][D / 32];  // double buffer (compile-time indexed)

  // where tile item i lives
  auto tile_src = [&](int i, int& Pn) -> const uint16_t* {
    const int bg = i / tiles_per_bg;
    const int L = c.seq_len[bg / c.Hkv];
    Pn = min((L + kPage - 1) / kPage, c.max_pages);
    return c.summary + (size_t)bg * c.max_pages * D;
  };
  auto compute = [&](int i, const uint4 (&av)[2][D / 32]) {
    const int bg = i / tiles_per_bg, tile = i % tiles_per_bg;
    if (bg != cur_bg) {  // new (b, g): its query fragments (hi + lo)
      cur_bg = bg;
      const int b = bg / c.Hkv, g = bg % c.Hkv;
      const int L = c.seq_len[b];
      P = min((L + kPage - 1) / kPage, c.max_pages);
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

  int Pn;
  const uint16_t* src = tile_src(i0, Pn);
  load_tile<D>(src, i0 % tiles_per_bg, Pn, lane, av0);
  for (int i = i0; i < i1; i += 2) {
    if (i + 1 < i1) {  // next tile into the odd buffer, then the even tile's math
      src = tile_src(i + 1, Pn);
      load_tile<D>(src, (i + 1) % tiles_per_bg, Pn, lane, av1);
    }
    compute(i, av0);
    if (i + 1 >= i1) break;
    if (i + 2 < i1) {
      src = tile_src(i + 2, Pn);
      load_tile<D>(src, (i + 2) % tiles_per_bg, Pn, lane, av0);
    }
    compute(i + 1, av1);
  }
  if (bad) set_err(c.err, KVQ_DERR_FP16_RANGE);
  griddep_launch_dependents();
}

template <int D, bool BF16>
cudaError_t launch_d(const DevCache& c, const void* q, float* scores, cudaStream_t s) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  const int tiles_per_bg = (c.max_pages + 15) / 16;
  const long long total = (long long)c.B * c.Hkv * tiles_per_bg;
  const long long blocks_max = 2LL * attn_num_ctas(dev);
  const long long warps = blocks_max * kScoreWarps;
  const int per = (int)((total + warps - 1) / warps);
  const long long blocks = (total + (long long)per * kScoreWarps - 1) / ((long long)per * kScoreWarps);
  return launch_pdl(score_kernel<D, BF16>, dim3((unsigned)blocks), dim3(kScoreWarps * 32), 0, s, c,
                    static_cast<const uint16_t*>(q), scores, tiles_per_bg, per);
}

}  // namespace

cudaError_t launch_scores(const DevCache& c, const void* q, float* scores, cudaStream_t s) {
  if (c.G > kMaxG) return cudaErrorInvalidValue;
  const bool bf = c.dtype == KVQ_DT_BF16;
  if (c.D == 128) return bf ? launch_d<128, true>(c, q, scores, s) : launch_d<128, false>(c, q, scores, s);
  if (c.D == 64) return bf ? launch_d<64, true>(c, q, scores, s) : launch_d<64, false>(c, q, scores, s);
  return cudaErrorInvalidValue;
}

}  // namespace kvq
