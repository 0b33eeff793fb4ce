// Page-score tile math shared by kvq_page_scores and the fused decode step.
//
// AMASS "decode-time sparse KV-cache attention for vLLM", "What is in the box": pages are
// ranked by a compact score computed from a tiny resident per-page summary.  Score of
// page p for kv head g: s[b][g][p] = max_{h in group g} sum_d q[b][h][d] * kbar[b][g][p][d].
//
// One warp scores a tile of 16 page summaries on the tensor core (mma m16n8k16, fp16
// inputs, fp32 accumulation): A = 16 summaries x 16 channels (fp16, as stored), B = the
// kv head's query rows (heads as N <= 8).  A bf16 query is split into an fp16 high part
// and an fp16 low part scaled by 2^24 (two mmas, the second accumulated apart and scaled
// back by 2^-24, a power of two): fp16 holds a bf16 value exactly from 2^-17 up to its
// range, and the scaled residual of a smaller one exactly down to 2^-41, so every product
// is exact for |q| >= 2^-41 (below that an element loses at most 2^-49 of its product's
// summary factor), as in an fp32 CUDA-core dot product.  An fp16 query is its own high
// part.  A 16-bit query element beyond the fp16 range is flagged (KVQ_DERR_FP16_RANGE).
// The channel order
// inside each k-step is permuted -- the same way for A and B, which leaves the dot
// product unchanged -- so that each lane reads its D/4 channels of a summary row as
// contiguous 16-byte loads from a row-major [page][D] layout (global or shared memory).
#pragma once

#include <math.h>

#include "kvq_internal.cuh"
#include "ptx.cuh"

namespace kvq {

// NaN-propagating max (a NaN score ranks lowest later; here it must survive the max)
__device__ inline float nanmax(float a, float b) { return (a != a || b != b) ? __int_as_float(0x7FC00000) : fmaxf(a, b); }

// The low part of a split query is stored times kQLoScale; its products are summed
// apart and multiplied by kQLoUnscale (both exact powers of two).
constexpr float kQLoScale = 0x1p24f;
constexpr float kQLoUnscale = 0x1p-24f;

// fp16 pair (hi) and scaled residual pair (lo = fp16((x - hi) * 2^24)) of two 16-bit query
// values; *bad if out of range.  x - hi is exact in fp32 (hi is x rounded, or 0).
template <bool BF16>
__device__ inline void split_q(uint32_t bits2, uint32_t& hi, uint32_t& lo, bool& bad) {
  const float x0 = bits_to_float<BF16>(static_cast<uint16_t>(bits2 & 0xFFFFu));
  const float x1 = bits_to_float<BF16>(static_cast<uint16_t>(bits2 >> 16));
  const __half2 h = __floats2half2_rn(x0, x1);
  const float2 hf = __half22float2(h);
  const __half2 l = __floats2half2_rn((x0 - hf.x) * kQLoScale, (x1 - hf.y) * kQLoScale);
  bad |= !(fabsf(x0) <= 65504.f) || !(fabsf(x1) <= 65504.f);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// Query fragments (hi + lo fp16 parts) of the G query heads of kv head g of sequence b.
template <int D, bool BF16>
struct QFrag {
  static constexpr int KS = D / 16;
  static constexpr int CW = D / 4;  // channels per lane per row
  uint32_t bh[KS][2], bl[KS][2];
  __device__ inline void load(const uint16_t* q, int Hq, int G, int b, int g, int lane, bool& bad) {
    const int g8 = lane >> 2, q4 = lane & 3;
    uint32_t w[CW / 2];
    if (g8 < G) {
      const uint4* src = reinterpret_cast<const uint4*>(q + ((size_t)b * Hq + (size_t)g * G + g8) * D + CW * q4);
#pragma unroll
      for (int k = 0; k < CW / 8; ++k) {
        const uint4 v = __ldcg(src + k);
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
};

// Lane's share of rows g8 and g8 + 8 of a 16-row summary tile starting at `rows` (row
// stride D): channels [CW*q4, CW*q4 + CW) of each row.
template <int D>
__device__ inline void load_tile_rows(const uint16_t* rows, int lane, uint4 (&av)[2][D / 32]) {
  constexpr int CW = D / 4;
  const int g8 = lane >> 2, q4 = lane & 3;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const uint4* src = reinterpret_cast<const uint4*>(rows + (size_t)(g8 + 8 * r) * D + CW * q4);
#pragma unroll
    for (int i = 0; i < CW / 8; ++i) av[r][i] = src[i];
  }
}

// Dot products of the tile's rows with the lane's two query heads: v[0] = (page g8, head
// 2q4), v[1] = (g8, 2q4 + 1), v[2] = (g8 + 8, 2q4), v[3] = (g8 + 8, 2q4 + 1).
template <int D, bool BF16>
__device__ inline void tile_head_dots(const uint4 (&av)[2][D / 32], const QFrag<D, BF16>& qf, float (&v)[4]) {
  constexpr int KS = D / 16;
  float ch[4] = {0.f, 0.f, 0.f, 0.f}, cl[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int kk = 0; kk < KS; ++kk) {
    // uint4 k holds k-steps 2k (.x = cols 2q4.., .y = cols 2q4+8..) and 2k+1 (.z, .w)
    const uint4 r0 = av[0][kk / 2];
    const uint4 r1 = av[1][kk / 2];
    const uint32_t a[4] = {(kk & 1) ? r0.z : r0.x, (kk & 1) ? r1.z : r1.x, (kk & 1) ? r0.w : r0.y,
                           (kk & 1) ? r1.w : r1.y};
    mma16816<false>(ch, a, qf.bh[kk][0], qf.bh[kk][1]);
    if constexpr (BF16) mma16816<false>(cl, a, qf.bl[kk][0], qf.bl[kk][1]);
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) v[j] = ch[j] + cl[j] * kQLoUnscale;
}

// Max over the lane's valid heads of values laid out as tile_head_dots's, then over the
// quad (NaN-propagating): m0 for row g8, m1 for row g8 + 8, valid in every lane of the quad.
__device__ inline void heads_max(const float (&v)[4], int G, int lane, float& m0, float& m1) {
  const int q4 = lane & 3;
  const bool h0ok = 2 * q4 < G, h1ok = 2 * q4 + 1 < G;
  m0 = nanmax(h0ok ? v[0] : -INFINITY, h1ok ? v[1] : -INFINITY);
  m1 = nanmax(h0ok ? v[2] : -INFINITY, h1ok ? v[3] : -INFINITY);
#pragma unroll
  for (int o = 1; o <= 2; o <<= 1) {
    m0 = nanmax(m0, __shfl_xor_sync(0xffffffffu, m0, o));
    m1 = nanmax(m1, __shfl_xor_sync(0xffffffffu, m1, o));
  }
}

// Scores of the tile's rows g8 (m0) and g8 + 8 (m1): max over the G heads, NaN-propagating;
// the result is valid in every lane of the row's quad.
template <int D, bool BF16>
__device__ inline void tile_scores(const uint4 (&av)[2][D / 32], const QFrag<D, BF16>& qf, int G, int lane,
                                   float& m0, float& m1) {
  float v[4];
  tile_head_dots<D, BF16>(av, qf, v);
  heads_max(v, G, lane, m0, m1);
}

}  // namespace kvq
