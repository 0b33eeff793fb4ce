// kvq_page_scores: page score from the mean-key summary.
//
// AMASS "decode-time sparse KV-cache attention for vLLM", "What is in the box": pages are
// ranked by a compact score computed from a tiny resident per-page summary; the score
// kernel is a bandwidth-bound sweep over all summaries.  Score of page p for kv head g:
//   s[b][g][p] = max_{h in group g} sum_d q[b][h][d] * kbar[b][g][p][d]
//
// The sweep runs on the tensor core (warp-level mma m16n8k16, fp16 inputs, fp32
// accumulation): A = 16 page summaries x 16 channels (fp16, as stored), B = the kv head's
// query rows (heads as N <= 8).  The query is split into fp16 hi + lo parts (two mmas),
// so every product is exact, as in an fp32 CUDA-core dot product; a 16-bit query element
// beyond the fp16 range is flagged (KVQ_DERR_FP16_RANGE).  The channel order inside each
// k-step is permuted -- the same way for A and B, which leaves the dot product unchanged --
// so that each lane reads its 32 channels of a summary row as four contiguous 16-byte loads
// (row-major [page][D] layout, no staging).  The summaries were prefetched into L2 by
// kvq_append when it ran just before.
#include <math.h>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kScoreWarps = 8;

// NaN-propagating max (a NaN score ranks lowest later; here it must survive the max)
__device__ inline float nanmax(float a, float b) { return (a != a || b != b) ? __int_as_float(0x7FC00000) : fmaxf(a, b); }

__device__ inline void mma_f16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// fp16 pair (hi) and residual pair (lo) of two 16-bit query values; *bad if out of range.
template <bool BF16>
__device__ inline void split_q(uint32_t bits2, uint32_t& hi, uint32_t& lo, bool& bad) {
  const float x0 = bits_to_float<BF16>(static_cast<uint16_t>(bits2 & 0xFFFFu));
  const float x1 = bits_to_float<BF16>(static_cast<uint16_t>(bits2 >> 16));
  const __half2 h = __floats2half2_rn(x0, x1);
  const float2 hf = __half22float2(h);
  const __half2 l = __floats2half2_rn(x0 - hf.x, x1 - hf.y);
  bad |= !(fabsf(x0) <= 65504.f) || !(fabsf(x1) <= 65504.f);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

template <int D, bool BF16>
__device__ inline void load_tile(const uint16_t* sbase, int tile, int P, int g8, uint4 (&av)[2][D / 32]) {
  constexpr int CW = D / 4;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int p = tile * 16 + g8 + 8 * r;
    const uint4* src = reinterpret_cast<const uint4*>(sbase + (size_t)p * D);
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
  constexpr int KS = D / 16;  // k-steps
  constexpr int CW = D / 4;   // channels per lane per row
  const int G = c.G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g8 = lane >> 2, q4 = lane & 3;
  const int total = c.B * c.Hkv * tiles_per_bg;
  const int i0 = (blockIdx.x * kScoreWarps + warp) * per;
  const int i1 = min(total, i0 + per);
  griddep_wait();
  if (i0 >= i1) return;
  const bool h0ok = 2 * q4 < G, h1ok = 2 * q4 + 1 < G;

  uint32_t bh[KS][2], bl[KS][2];
  int cur_bg = -1, P = 0;
  float* out = nullptr;
  bool bad = false;
  uint4 av0[2][D / 32], av1[2][D / 32];  // double buffer (compile-time indexed)

  // where tile item i lives
  auto tile_src = [&](int i, int& Pn) -> const uint16_t* {
    const int bg = i / tiles_per_bg;
    const int L = c.seq_len[bg / c.Hkv];
    Pn = min((L + kPage - 1) / kPage, c.max_pages);
    return c.summary + (size_t)bg * c.max_pages * D + CW * q4;
  };
  auto compute = [&](int i, const uint4 (&av)[2][D / 32]) {
    const int bg = i / tiles_per_bg, tile = i % tiles_per_bg;
    if (bg != cur_bg) {  // new (b, g): its query fragments (hi + lo)
      cur_bg = bg;
      const int b = bg / c.Hkv, g = bg % c.Hkv;
      const int L = c.seq_len[b];
      P = min((L + kPage - 1) / kPage, c.max_pages);
      out = scores + (size_t)bg * c.max_pages;
      uint32_t w[CW / 2];
      if (g8 < G) {
        const uint4* src = reinterpret_cast<const uint4*>(q + ((size_t)b * c.Hq + (size_t)g * G + g8) * D + CW * q4);
#pragma unroll
        for (int k = 0; k < CW / 8; ++k) {
          const uint4 v = src[k];
          w[4 * k] = v.x; w[4 * k + 1] = v.y; w[4 * k + 2] = v.z; w[4 * k + 3] = v.w;
        }
      } else {
#pragma unroll
        for (int k = 0; k < CW / 2; ++k) w[k] = 0u;
      }
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
        split_q<BF16>(w[2 * kk], bh[kk][0], bl[kk][0], bad);
        split_q<BF16>(w[2 * kk + 1], bh[kk][1], bl[kk][1], bad);
      }
    }
    float ch[4] = {0.f, 0.f, 0.f, 0.f}, cl[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      // uint4 k holds k-steps 2k (.x = cols 2q4.., .y = cols 2q4+8..) and 2k+1 (.z, .w)
      const uint4 r0 = av[0][kk / 2];
      const uint4 r1 = av[1][kk / 2];
      const uint32_t a[4] = {(kk & 1) ? r0.z : r0.x, (kk & 1) ? r1.z : r1.x, (kk & 1) ? r0.w : r0.y,
                             (kk & 1) ? r1.w : r1.y};
      mma_f16(ch, a, bh[kk][0], bh[kk][1]);
      if constexpr (BF16) mma_f16(cl, a, bl[kk][0], bl[kk][1]);
    }
    // c: (page g8, head 2q4), (g8, 2q4+1), (g8 + 8, 2q4), (g8 + 8, 2q4+1)
    const float v0 = h0ok ? ch[0] + cl[0] : -INFINITY, v1 = h1ok ? ch[1] + cl[1] : -INFINITY;
    const float v2 = h0ok ? ch[2] + cl[2] : -INFINITY, v3 = h1ok ? ch[3] + cl[3] : -INFINITY;
    float m0 = nanmax(v0, v1), m1 = nanmax(v2, v3);
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      m0 = nanmax(m0, __shfl_xor_sync(0xffffffffu, m0, o));
      m1 = nanmax(m1, __shfl_xor_sync(0xffffffffu, m1, o));
    }
    if (q4 == 0) {
      const int p0 = tile * 16 + g8, p1 = p0 + 8;
      if (p0 < c.max_pages) out[p0] = p0 < P ? m0 : -INFINITY;
      if (p1 < c.max_pages) out[p1] = p1 < P ? m1 : -INFINITY;
    }
  };

  int Pn;
  const uint16_t* src = tile_src(i0, Pn);
  load_tile<D, BF16>(src, i0 % tiles_per_bg, Pn, g8, av0);
  for (int i = i0; i < i1; i += 2) {
    if (i + 1 < i1) {  // next tile into the odd buffer, then the even tile's math
      src = tile_src(i + 1, Pn);
      load_tile<D, BF16>(src, (i + 1) % tiles_per_bg, Pn, g8, av1);
    }
    compute(i, av0);
    if (i + 1 >= i1) break;
    if (i + 2 < i1) {
      src = tile_src(i + 2, Pn);
      load_tile<D, BF16>(src, (i + 2) % tiles_per_bg, Pn, g8, av0);
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
