// kvq_page_scores: page score from the mean-key summary.
//
// AMASS "decode-time sparse KV-cache attention for vLLM", "What is in the box": pages are
// ranked by a compact score computed from a tiny resident per-page summary; the score
// kernel is a bandwidth-bound sweep over all summaries.  Score of page p for kv head g:
//   s[b][g][p] = max_{h in group g} sum_d q[b][h][d] * kbar[b][g][p][d]
// in fp32 (products of a 16-bit query element and an fp16 summary element are exact in
// fp32; the sum is an 8-element chain per lane followed by a butterfly tree).
//
// Mapping: D/8 lanes per page, 8 channels (one 16-byte load) per lane, the kv head's G
// query rows held in registers; each warp sweeps 16 consecutive pages of one (b, g).
#include <math.h>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kScoreWarps = 8;
constexpr int kScoreIters = 8;

__device__ inline void unpack8(const uint4& v, float (&f)[8], bool bf16) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (bf16) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    } else {
      const float2 t = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
}

template <int D, int G, bool BF16>
__global__ void __launch_bounds__(kScoreWarps * 32) score_kernel(DevCache c, const uint16_t* __restrict__ q,
                                                                 float* __restrict__ scores) {
  constexpr int LPP = D / 8;    // lanes per page
  constexpr int PPI = 32 / LPP; // pages per warp iteration
  constexpr int PPW = PPI * kScoreIters;
  const int bg = blockIdx.y;
  const int b = bg / c.Hkv, g = bg % c.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane % LPP, pp = lane / LPP;
  const int p0 = (blockIdx.x * kScoreWarps + warp) * PPW;
  if (p0 >= c.max_pages) return;
  const int L = c.seq_len[b];
  const int P = min((L + kPage - 1) / kPage, c.max_pages);

  float qr[G][8];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const uint4 v = *reinterpret_cast<const uint4*>(q + ((size_t)b * c.Hq + (size_t)g * G + h) * D + sub * 8);
    unpack8(v, qr[h], BF16);
  }
  const uint16_t* srow = c.summary + (size_t)bg * c.max_pages * D + sub * 8;
  float* out = scores + (size_t)bg * c.max_pages;

#pragma unroll 2
  for (int it = 0; it < kScoreIters; ++it) {
    const int p = p0 + it * PPI + pp;
    const bool valid = p < P;
    float acc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) acc[h] = 0.f;
    if (valid) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(srow + (size_t)p * D));
      float k[8];
      unpack8(v, k, false);  // summaries are fp16
#pragma unroll
      for (int h = 0; h < G; ++h) {
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[h] = fmaf(qr[h][e], k[e], acc[h]);
      }
    }
#pragma unroll
    for (int o = LPP / 2; o >= 1; o >>= 1) {
#pragma unroll
      for (int h = 0; h < G; ++h) acc[h] += __shfl_xor_sync(0xffffffffu, acc[h], o);
    }
    float s = acc[0];
#pragma unroll
    for (int h = 1; h < G; ++h) s = (isnan(s) || acc[h] <= s) ? s : acc[h];
#pragma unroll
    for (int h = 1; h < G; ++h) s = isnan(acc[h]) ? acc[h] : s;
    if (sub == 0 && p < c.max_pages) out[p] = valid ? s : -INFINITY;
  }
}

template <int D, bool BF16>
cudaError_t launch_d(const DevCache& c, const void* q, float* scores, cudaStream_t s) {
  constexpr int PPB = (32 / (D / 8)) * kScoreIters * kScoreWarps;
  const dim3 grid((c.max_pages + PPB - 1) / PPB, c.B * c.Hkv);
  const uint16_t* qq = static_cast<const uint16_t*>(q);
  switch (c.G) {
    case 1: score_kernel<D, 1, BF16><<<grid, kScoreWarps * 32, 0, s>>>(c, qq, scores); break;
    case 2: score_kernel<D, 2, BF16><<<grid, kScoreWarps * 32, 0, s>>>(c, qq, scores); break;
    case 4: score_kernel<D, 4, BF16><<<grid, kScoreWarps * 32, 0, s>>>(c, qq, scores); break;
    case 8: score_kernel<D, 8, BF16><<<grid, kScoreWarps * 32, 0, s>>>(c, qq, scores); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_scores(const DevCache& c, const void* q, float* scores, cudaStream_t s) {
  const bool bf = c.dtype == KVQ_DT_BF16;
  if (c.D == 128) return bf ? launch_d<128, true>(c, q, scores, s) : launch_d<128, false>(c, q, scores, s);
  if (c.D == 64) return bf ? launch_d<64, true>(c, q, scores, s) : launch_d<64, false>(c, q, scores, s);
  return cudaErrorInvalidValue;
}

}  // namespace kvq
