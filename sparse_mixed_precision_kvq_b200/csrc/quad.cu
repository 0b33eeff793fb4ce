// quad page score: kvq_quad_build, kvq_quad_append, kvq_quad_page_scores and
// kvq_quad_append_scores (the token append, the quad state update and the scores in one
// launch).
//
// AMASS "decode-time sparse KV-cache attention for vLLM", "What is in the box", Stage A:
// a quadratic, Gaussian-MGF page score built from a tiny per-page summary that keeps r'
// eigenvalues per page.  Reading (the page gives no formula, rank or basis): with the
// caller's orthonormal basis rows u_i of a kv head, page p keeps
// lambda[p][i] = u_i^T Sigma_p u_i, the (1/n) variance of its keys along u_i, and scores
//   max_h  s q_h.kbar_p + 1/2 s^2 sum_i lambda[p][i] (u_i.q_h)^2,
// the log of the Gaussian moment-generating function E[exp(s q.k)] for k ~ N(kbar_p,
// Sigma_p) restricted to the basis.
//
// State arithmetic is IEEE fp64 without fused multiply-add (this unit is compiled with
// -fmad=false): y_i = sum_d u[i][d] k[d] in channel order, S1 = sum_t y and S2 = sum_t y^2
// in token order, lambda = fp16(max(S2/n - (S1/n)^2, 0)); a page built at once and a page
// grown token by token hold the same bits.  The score is fp32: the q.kbar part on the
// tensor core exactly as kvq_page_scores (score_tile.cuh), (u_i.q_h)^2 on the tensor core
// once per (sequence, kv head) and warp, the quadratic sum on the CUDA cores.
#include <math.h>

#include "kvq_internal.cuh"
#include "ptx.cuh"
#include "quant.cuh"
#include "score_tile.cuh"
#include "tile_split.cuh"

namespace kvq {
namespace {

template <bool BF16>
__device__ inline double key_f64(uint16_t v) {
  return static_cast<double>(bits_to_float<BF16>(v));
}

__device__ inline uint16_t quad_lambda(double s1, double s2, int n, bool& ov) {
  const double m = s1 / static_cast<double>(n);
  double v = s2 / static_cast<double>(n) - m * m;
  v = v > 0.0 ? v : 0.0;
  return fp16_sat(v, ov);
}

// One CTA per (page, sequence * kv head) of the prefilled context.
template <bool BF16>
__global__ void __launch_bounds__(256) quad_build_kernel(DevCache c, DevQuad qd, const uint16_t* __restrict__ ksrc,
                                                         const int64_t* __restrict__ cu, int64_t src_tokens) {
  const int p = blockIdx.x, bg = blockIdx.y;
  const int b = bg / c.Hkv, g = bg % c.Hkv;
  const int D = c.D, r = qd.rank, tid = threadIdx.x;
  const int L = c.seq_len[b];
  const int P = (L + kPage - 1) / kPage;
  if (p >= P || p >= c.max_pages) return;
  const int n = min(kPage, L - p * kPage);
  const int64_t row0 = cu[b] + (int64_t)p * kPage;
  if (row0 < 0 || row0 + n > src_tokens) {
    if (tid == 0) set_err(c.err, KVQ_DERR_BAD_POS);
    return;
  }
  __shared__ float ub[kMaxQuadRank * 128];  // basis rows of kv head g
  __shared__ uint16_t kb[kPage * 128];      // the page's keys
  __shared__ double ys[kPage][kMaxQuadRank + 1];
  for (int i = tid; i < r * D; i += blockDim.x) ub[i] = qd.basis[(size_t)g * r * D + i];
  for (int i = tid; i < n * D; i += blockDim.x) {
    const int t = i / D, d = i % D;
    kb[i] = ksrc[((size_t)g * src_tokens + (size_t)(row0 + t)) * D + d];
  }
  __syncthreads();
  for (int e = tid; e < n * r; e += blockDim.x) {
    const int t = e / r, i = e % r;
    double y = 0.0;
    for (int d = 0; d < D; ++d) y = y + static_cast<double>(ub[i * D + d]) * key_f64<BF16>(kb[t * D + d]);
    ys[t][i] = y;
  }
  __syncthreads();
  if (tid < r) {
    double s1 = 0.0, s2 = 0.0;
    for (int t = 0; t < n; ++t) {
      const double y = ys[t][tid];
      s1 = s1 + y;
      s2 = s2 + y * y;
    }
    bool ov = false;
    qd.lambda[((size_t)bg * c.max_pages + p) * r + tid] = quad_lambda(s1, s2, n, ov);
    if (p == P - 1) {
      double* o = qd.open + (size_t)bg * 2 * r;
      o[tid] = (L % kPage) ? s1 : 0.0;
      o[r + tid] = (L % kPage) ? s2 : 0.0;
    }
    if (ov) set_err(c.err, KVQ_DERR_FP16_RANGE);
  }
}

// One warp: token `pos` (0 <= pos < max_pages * 16) of sequence b, kv head g, key `krow`,
// joins the quad state; lane i < r owns basis row i.  The dot product is a sequential fp64
// chain over the channels; the basis row and the key are fetched 8 channels ahead of it.
template <int D, bool BF16>
__device__ inline void quad_append_warp(const DevCache& c, const DevQuad& qd, int bg, int g, int ps,
                                        const uint16_t* krow, int lane) {
  const int r = qd.rank;
  if (lane >= r) return;
  const int p = ps / kPage, t = ps % kPage;
  const float4* u4 = reinterpret_cast<const float4*>(qd.basis + ((size_t)g * r + lane) * D);
  double y = 0.0;
#pragma unroll
  for (int c8 = 0; c8 < D / 8; ++c8) {
    const float4 ua = u4[2 * c8], ub = u4[2 * c8 + 1];
    const float uu[8] = {ua.x, ua.y, ua.z, ua.w, ub.x, ub.y, ub.z, ub.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) y = y + static_cast<double>(uu[j]) * key_f64<BF16>(krow[8 * c8 + j]);
  }
  double* o = qd.open + (size_t)bg * 2 * r;
  const double s1 = t == 0 ? y : o[lane] + y;
  const double s2 = t == 0 ? y * y : o[r + lane] + y * y;
  o[lane] = s1;
  o[r + lane] = s2;
  bool ov = false;
  qd.lambda[((size_t)bg * c.max_pages + p) * r + lane] = quad_lambda(s1, s2, t + 1, ov);
  if (ov) set_err(c.err, KVQ_DERR_FP16_RANGE);
}

// One warp per (sequence, kv head).
template <int D, bool BF16>
__global__ void __launch_bounds__(32) quad_append_kernel(DevCache c, DevQuad qd, const int32_t* __restrict__ pos,
                                                         const uint16_t* __restrict__ k_new) {
  const int bg = blockIdx.x, b = bg / c.Hkv, g = bg % c.Hkv, lane = threadIdx.x;
  griddep_wait();
  const int ps = pos[b];
  if (ps >= 0 && ps >= c.max_pages * kPage) {
    if (lane == 0 && g == 0) set_err(c.err, KVQ_DERR_BAD_POS);
  } else if (ps >= 0) {
    quad_append_warp<D, BF16>(c, qd, bg, g, ps, k_new + (size_t)bg * D, lane);
  }
  griddep_launch_dependents();
}

// zs[h][i] = (u_i . q_h)^2 for the query heads of kv head g, on the tensor core: A = 16
// basis rows (fp32 split into fp16 hi + lo parts) in the permuted channel order of the
// score tile (lane (g8, q4) loads channels [D/4 q4, D/4 q4 + D/4) of rows g8 and g8 + 8 as
// 16-byte loads), B = the query fragments already in registers (hi + lo), fp32
// accumulation: u_hi q_hi + u_lo q_hi + u_hi q_lo, all products exact.  Rows past the rank
// load as zero; heads past G are zero rows of B, so their terms are 0.
__device__ inline void split_f32x2(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(a, b);
  const float2 hf = __half22float2(h);
  const __half2 l = __floats2half2_rn(a - hf.x, b - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

template <int D, bool BF16>
__device__ inline void quad_qterms(const DevQuad& qd, const QFrag<D, BF16>& qf, int g, int lane,
                                   float (*zs)[kMaxQuadRank]) {
  constexpr int KS = D / 16, CW = D / 4;
  const int g8 = lane >> 2, q4 = lane & 3;
  const float* ub = qd.basis + (size_t)g * qd.rank * D + CW * q4;
  for (int m0 = 0; m0 < qd.rank; m0 += 16) {
    const int i0 = m0 + g8, i1 = m0 + g8 + 8;
    const bool ok0 = i0 < qd.rank, ok1 = i1 < qd.rank;
    const float4* s0 = reinterpret_cast<const float4*>(ub + (size_t)i0 * D);
    const float4* s1 = reinterpret_cast<const float4*>(ub + (size_t)i1 * D);
    float4 x0[KS], x1[KS];
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      x0[kk] = ok0 ? s0[kk] : make_float4(0.f, 0.f, 0.f, 0.f);
      x1[kk] = ok1 ? s1[kk] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float cacc[4] = {0.f, 0.f, 0.f, 0.f}, clo[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      uint32_t ah[4], al[4];
      split_f32x2(x0[kk].x, x0[kk].y, ah[0], al[0]);
      split_f32x2(x1[kk].x, x1[kk].y, ah[1], al[1]);
      split_f32x2(x0[kk].z, x0[kk].w, ah[2], al[2]);
      split_f32x2(x1[kk].z, x1[kk].w, ah[3], al[3]);
      mma16816<false>(cacc, ah, qf.bh[kk][0], qf.bh[kk][1]);
      mma16816<false>(cacc, al, qf.bh[kk][0], qf.bh[kk][1]);
      if constexpr (BF16) mma16816<false>(clo, ah, qf.bl[kk][0], qf.bl[kk][1]);  // query low part, x 2^24
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) cacc[j] += clo[j] * kQLoUnscale;
    // cacc: (row i0, head 2 q4), (i0, 2 q4 + 1), (i1, 2 q4), (i1, 2 q4 + 1)
    if (ok0) {
      zs[2 * q4][i0] = cacc[0] * cacc[0];
      zs[2 * q4 + 1][i0] = cacc[1] * cacc[1];
    }
    if (ok1) {
      zs[2 * q4][i1] = cacc[2] * cacc[2];
      zs[2 * q4 + 1][i1] = cacc[3] * cacc[3];
    }
  }
  __syncwarp();
}

constexpr int kQuadWarps = 8;

template <int D, int RK>
__device__ inline void quad_load_tile(const uint16_t* sbase, const uint16_t* lbase, int tile, int P, int lane,
                                      uint4 (&av)[2][D / 32], uint4 (&lv)[2][RK]) {
  constexpr int CW = D / 4;
  const int g8 = lane >> 2, q4 = lane & 3;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int p = tile * 16 + g8 + 8 * h;
    const uint4* src = reinterpret_cast<const uint4*>(sbase + (size_t)p * D + CW * q4);
#pragma unroll
    for (int i = 0; i < CW / 8; ++i) av[h][i] = p < P ? __ldcg(src + i) : make_uint4(0, 0, 0, 0);
    const uint4* ls = reinterpret_cast<const uint4*>(lbase + (size_t)p * 8 * RK);
#pragma unroll
    for (int k = 0; k < RK; ++k) lv[h][k] = p < P ? __ldcg(ls + k) : make_uint4(0, 0, 0, 0);
  }
}

// Warp w takes a contiguous run of the flat list of 16-page tiles, as kvq_page_scores
// does -- REAL: only the tiles that hold pages, divided evenly (tile_split.cuh); else
// [w * per, (w + 1) * per) of every row's max_pages / 16 tiles -- loading the next tile
// (summary rows and lambda rows) while the current one is multiplied; the two buffers
// take more registers than two CTAs per SM leave, so one CTA of 8 warps runs per SM.
// With `ap.pos` set (kvq_quad_append_scores) the warp that owns the tile of a (b, g)'s
// appended token first writes the token into the cache (quantise, pack, summary) and the
// quad state, so that tile is read after both are stored.
struct QuadAppend {
  const int32_t* pos;  // nullable: no append
  const uint16_t* k_new;
  const uint16_t* v_new;
};

template <int D, bool BF16, int RK, bool REAL>
__global__ void __launch_bounds__(kQuadWarps * 32, 1)
    quad_score_kernel(DevCache c, DevQuad qd, const uint16_t* __restrict__ q, float sm_scale,
                      float* __restrict__ scores, int tiles_per_bg, int per, QuadAppend ap) {
  extern __shared__ __align__(16) int pre[];             // REAL: the tile prefix [B * Hkv + 1]
  __shared__ float zs[kQuadWarps][kMaxG][kMaxQuadRank];  // (u_i . q_h)^2 of the warp's current (b, g)
  __shared__ int s_part[kQuadWarps];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, q4 = lane & 3;
  const int r = qd.rank;
  const int BH = c.B * c.Hkv;
  const int nw = gridDim.x * kQuadWarps, gw = blockIdx.x * kQuadWarps + warp;
  int total, i0, i1;
  if constexpr (REAL) {  // (no append: the owner of an appended tile is defined on whole rows)
    total = row_tile_prefix<kQuadWarps * 32>(c, pre, s_part, tid);
    const int pw = (total + nw - 1) / nw;
    i0 = min(total, gw * pw);
    i1 = min(total, i0 + pw);
  } else {
    total = BH * tiles_per_bg;
    i0 = gw * per;
    i1 = min(total, i0 + per);
  }
  griddep_wait();
  if constexpr (REAL) fill_past_tiles(c, pre, scores, gw, nw, lane);
  if (!REAL && ap.pos != nullptr && i0 < i1) {  // appends whose page lies in this warp's tiles
    for (int bg = i0 / tiles_per_bg; bg <= (i1 - 1) / tiles_per_bg; ++bg) {
      const int b = bg / c.Hkv, g = bg % c.Hkv;
      const int ps = ap.pos[b];
      if (ps < 0) continue;
      if (ps >= c.max_pages * kPage) {
        if (lane == 0 && g == 0 && bg * tiles_per_bg >= i0) set_err(c.err, KVQ_DERR_BAD_POS);
        continue;
      }
      const int it = bg * tiles_per_bg + (ps / kPage) / 16;
      if (it < i0 || it >= i1) continue;
      append_token_warp<BF16>(c, b, g, ps, ap.k_new + (size_t)bg * D, ap.v_new + (size_t)bg * D, lane, nullptr);
      quad_append_warp<D, BF16>(c, qd, bg, g, ps, ap.k_new + (size_t)bg * D, lane);
      __syncwarp();
    }
  }
  if (i0 < i1) {
    const float c1 = sm_scale, c2 = 0.5f * sm_scale * sm_scale;
    QFrag<D, BF16> qf;
    int cur_bg = -1, P = 0;
    float* out = nullptr;
    bool bad = false;
    uint4 av0[2][D / 32], av1[2][D / 32];
    uint4 lv0[2][RK], lv1[2][RK];

    int lcur = REAL ? row_of_item(pre, BH, i0) : 0, ccur = lcur;  // forward cursors (REAL)
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
    auto load = [&](int i, uint4 (&av)[2][D / 32], uint4 (&lv)[2][RK]) {
      int tile;
      const int bg = locate(i, lcur, tile);
      const int Pn = row_pages(c, bg);
      quad_load_tile<D, RK>(c.summary + (size_t)bg * c.max_pages * D, qd.lambda + (size_t)bg * c.max_pages * r,
                            tile, Pn, lane, av, lv);
    };
    auto compute = [&](int i, const uint4 (&av)[2][D / 32], const uint4 (&lv)[2][RK]) {
      int tile;
      const int bg = locate(i, ccur, tile);
      if (bg != cur_bg) {  // new (b, g): query fragments and (u_i . q_h)^2
        cur_bg = bg;
        const int b = bg / c.Hkv, g = bg % c.Hkv;
        P = row_pages(c, bg);
        out = scores + (size_t)bg * c.max_pages;
        qf.load(q, c.Hq, c.G, b, g, lane, bad);
        quad_qterms<D, BF16>(qd, qf, g, lane, zs[warp]);
        __syncwarp();
      }
      float v[4];
      tile_head_dots<D, BF16>(av, qf, v);
      float qs[4] = {0.f, 0.f, 0.f, 0.f};
      const float* z0 = zs[warp][(2 * q4) & (kMaxG - 1)];
      const float* z1 = zs[warp][(2 * q4 + 1) & (kMaxG - 1)];
#pragma unroll
      for (int k = 0; k < RK; ++k) {
        {
          const uint32_t w0[4] = {lv[0][k].x, lv[0][k].y, lv[0][k].z, lv[0][k].w};
          const uint32_t w1[4] = {lv[1][k].x, lv[1][k].y, lv[1][k].z, lv[1][k].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 l0 = __half22float2(*reinterpret_cast<const __half2*>(&w0[e]));
            const float2 l1 = __half22float2(*reinterpret_cast<const __half2*>(&w1[e]));
            const int i = 8 * k + 2 * e;
            qs[0] = fmaf(l0.x, z0[i], fmaf(l0.y, z0[i + 1], qs[0]));
            qs[1] = fmaf(l0.x, z1[i], fmaf(l0.y, z1[i + 1], qs[1]));
            qs[2] = fmaf(l1.x, z0[i], fmaf(l1.y, z0[i + 1], qs[2]));
            qs[3] = fmaf(l1.x, z1[i], fmaf(l1.y, z1[i + 1], qs[3]));
          }
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = c1 * v[j] + c2 * qs[j];
      float m0, m1;
      heads_max(v, c.G, lane, m0, m1);
      if (q4 == 0) {
        const int p0 = tile * 16 + g8, p1 = p0 + 8;
        if (p0 < c.max_pages) out[p0] = p0 < P ? m0 : -INFINITY;
        if (p1 < c.max_pages) out[p1] = p1 < P ? m1 : -INFINITY;
      }
    };

    load(i0, av0, lv0);
    for (int i = i0; i < i1; i += 2) {
      if (i + 1 < i1) load(i + 1, av1, lv1);
      compute(i, av0, lv0);
      if (i + 1 >= i1) break;
      if (i + 2 < i1) load(i + 2, av0, lv0);
      compute(i + 1, av1, lv1);
    }
    if (bad) set_err(c.err, KVQ_DERR_FP16_RANGE);
  }
  griddep_launch_dependents();
}

template <int D, bool BF16, int RK>
cudaError_t launch_quad_scores_r(const DevCache& c, const DevQuad& qd, const void* q, float sm_scale, float* scores,
                                 const QuadAppend& ap, cudaStream_t s) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  const int tiles_per_bg = (c.max_pages + 15) / 16;
  const long long total = (long long)c.B * c.Hkv * tiles_per_bg;
  const long long warps = (long long)sm_count(dev) * kQuadWarps;  // one CTA per SM (registers)
  const int per = (int)((total + warps - 1) / warps);
  const long long blocks = (total + (long long)per * kQuadWarps - 1) / ((long long)per * kQuadWarps);
  const size_t smem = ((size_t)c.B * c.Hkv + 1) * sizeof(int);
  if (ap.pos == nullptr && smem <= 32 * 1024)  // the tile prefix beside the 8 KB of (u_i . q_h)^2
    return launch_pdl(quad_score_kernel<D, BF16, RK, true>, dim3((unsigned)blocks), dim3(kQuadWarps * 32), smem, s,
                      c, qd, static_cast<const uint16_t*>(q), sm_scale, scores, tiles_per_bg, per, ap);
  return launch_pdl(quad_score_kernel<D, BF16, RK, false>, dim3((unsigned)blocks), dim3(kQuadWarps * 32), 0, s, c,
                    qd, static_cast<const uint16_t*>(q), sm_scale, scores, tiles_per_bg, per, ap);
}

template <int D, bool BF16>
cudaError_t launch_quad_scores_d(const DevCache& c, const DevQuad& qd, const void* q, float sm_scale, float* scores,
                                 const QuadAppend& ap, cudaStream_t s) {
  switch (qd.rank / 8) {
    case 1: return launch_quad_scores_r<D, BF16, 1>(c, qd, q, sm_scale, scores, ap, s);
    case 2: return launch_quad_scores_r<D, BF16, 2>(c, qd, q, sm_scale, scores, ap, s);
    case 3: return launch_quad_scores_r<D, BF16, 3>(c, qd, q, sm_scale, scores, ap, s);
    case 4: return launch_quad_scores_r<D, BF16, 4>(c, qd, q, sm_scale, scores, ap, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_quad_build(const DevCache& c, const DevQuad& qd, const void* k_src, const int64_t* cu,
                              int64_t src_tokens, cudaStream_t s) {
  const dim3 grid(c.max_pages, c.B * c.Hkv);
  const uint16_t* k = static_cast<const uint16_t*>(k_src);
  if (c.dtype == KVQ_DT_BF16) quad_build_kernel<true><<<grid, 256, 0, s>>>(c, qd, k, cu, src_tokens);
  else quad_build_kernel<false><<<grid, 256, 0, s>>>(c, qd, k, cu, src_tokens);
  return cudaGetLastError();
}

cudaError_t launch_quad_append(const DevCache& c, const DevQuad& qd, const int32_t* pos, const void* k_new,
                               cudaStream_t s) {
  const uint16_t* k = static_cast<const uint16_t*>(k_new);
  const dim3 grid(c.B * c.Hkv);
  const bool bf = c.dtype == KVQ_DT_BF16;
  if (c.D == 128)
    return bf ? launch_pdl(quad_append_kernel<128, true>, grid, dim3(32), 0, s, c, qd, pos, k)
              : launch_pdl(quad_append_kernel<128, false>, grid, dim3(32), 0, s, c, qd, pos, k);
  return bf ? launch_pdl(quad_append_kernel<64, true>, grid, dim3(32), 0, s, c, qd, pos, k)
            : launch_pdl(quad_append_kernel<64, false>, grid, dim3(32), 0, s, c, qd, pos, k);
}

cudaError_t launch_quad_scores(const DevCache& c, const DevQuad& qd, const void* q, float sm_scale, float* scores,
                               const int32_t* pos, const void* k_new, const void* v_new, cudaStream_t s) {
  if (c.G > kMaxG) return cudaErrorInvalidValue;
  const bool bf = c.dtype == KVQ_DT_BF16;
  const QuadAppend ap{pos, static_cast<const uint16_t*>(k_new), static_cast<const uint16_t*>(v_new)};
  if (c.D == 128)
    return bf ? launch_quad_scores_d<128, true>(c, qd, q, sm_scale, scores, ap, s)
              : launch_quad_scores_d<128, false>(c, qd, q, sm_scale, scores, ap, s);
  if (c.D == 64)
    return bf ? launch_quad_scores_d<64, true>(c, qd, q, sm_scale, scores, ap, s)
              : launch_quad_scores_d<64, false>(c, qd, q, sm_scale, scores, ap, s);
  return cudaErrorInvalidValue;
}

}  // namespace kvq
