// Quantise-and-pack: kvq_append (one token per sequence) and kvq_build_pages (whole pages).
//
// Tiers after ARGUS "Virtual Memory for Transformers", "The One-Minute Explanation" and
// "Visual Architecture": 16-bit hot pages; INT8, INT4 (two per byte), INT2 (four per
// byte) and 1-bit (eight per byte) cold pages.  Quantiser, per 32-channel group of one
// token: zero = fp16(min), scale = fp16((max - min) / (2^b - 1)),
// code = clamp(rint((x - zero) / scale), 0, 2^b - 1) (0 when scale == 0); 1-bit: sign
// (x >= 0) and fp16(sum|x| / 32) summed in channel order.  Every step is an IEEE binary64
// operation with round-half-even, so the bytes do not depend on the thread mapping.
// The per-page mean-key summary (AMASS "What is in the box": a tiny per-page summary)
// is fp16(S / n) with S the fp64 sum of the page's keys in token order.
#include "kvq_internal.cuh"

namespace kvq {
namespace {

struct QOut {
  uint32_t code;
  uint32_t meta;  // INT-b: scale | zero << 16 ; 1-bit: magnitude
};

// Warp-collective: lane j holds channel j of the group.
__device__ inline QOut quant_group(double x, int tier, bool& ov) {
  const unsigned full = 0xffffffffu;
  if (tier == KVQ_TIER_I1) {
    const uint32_t bit = (x >= 0.0) ? 1u : 0u;
    const double ax = fabs(x);
    double s = 0.0;
#pragma unroll
    for (int j = 0; j < kGroup; ++j) s += __shfl_sync(full, ax, j);
    const uint16_t m = fp16_sat(s / 32.0, ov);
    return {bit, m};
  }
  double lo = x, hi = x;
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    lo = fmin(lo, __shfl_xor_sync(full, lo, o));
    hi = fmax(hi, __shfl_xor_sync(full, hi, o));
  }
  const double qmax = static_cast<double>((1 << tier_bits(tier)) - 1);
  const uint16_t zb = fp16_sat(lo, ov);
  const uint16_t sb = fp16_sat((hi - lo) / qmax, ov);
  const double zero = static_cast<double>(__half2float(__ushort_as_half(zb)));
  const double scale = static_cast<double>(__half2float(__ushort_as_half(sb)));
  uint32_t code = 0;
  if (scale != 0.0) {
    double c = rint((x - zero) / scale);
    c = fmin(fmax(c, 0.0), qmax);
    code = static_cast<uint32_t>(c);
  }
  return {code, static_cast<uint32_t>(sb) | (static_cast<uint32_t>(zb) << 16)};
}

template <bool BF16>
__device__ inline double to_double(uint16_t v) {
  return static_cast<double>(bits_to_float<BF16>(v));
}

// ----------------------------------------------------------------------------- append
template <bool BF16>
__global__ void __launch_bounds__(128) append_kernel(DevCache c, const int32_t* __restrict__ pos,
                                                     const uint16_t* __restrict__ k_new,
                                                     const uint16_t* __restrict__ v_new) {
  const int bg = blockIdx.x;
  const int b = bg / c.Hkv, g = bg % c.Hkv;
  const int D = c.D;
  const int tid = threadIdx.x;
  griddep_wait();
  const int P = pos[b];
  if (P < 0) return;
  if (P >= c.max_pages * kPage) {
    if (tid == 0) set_err(c.err, KVQ_DERR_BAD_POS);
    return;
  }
  const int page = P / kPage, t = P % kPage;
  int tier;
  const unsigned char* ck;
  if (!page_chunk(c, b, page, g, tier, ck)) return;
  unsigned char* chunk[2] = {const_cast<unsigned char*>(ck), const_cast<unsigned char*>(ck) + c.chunk[tier]};

  __shared__ double xs[2][128];
  __shared__ uint16_t xb[2][128];
  __shared__ uint32_t codes[2][128];
  __shared__ uint32_t metas[2][4];
  bool ov = false, nonfinite = false;

  if (tid < D) {
    xb[0][tid] = k_new[(size_t)bg * D + tid];
    xb[1][tid] = v_new[(size_t)bg * D + tid];
    xs[0][tid] = to_double<BF16>(xb[0][tid]);
    xs[1][tid] = to_double<BF16>(xb[1][tid]);
    nonfinite = !isfinite(xs[0][tid]) || !isfinite(xs[1][tid]);
    // running key sum of the open page and the page summary
    double* ks = c.open_ksum + (size_t)bg * D + tid;
    const double S = (t == 0) ? xs[0][tid] : (*ks + xs[0][tid]);
    *ks = S;
    c.summary[((size_t)bg * c.max_pages + page) * D + tid] = fp16_sat(S / static_cast<double>(t + 1), ov);
  }
  if (t == 0) {  // a newly opened page starts from zero bytes
    uint4* p4 = reinterpret_cast<uint4*>(chunk[0]);
    const int n16 = 2 * c.chunk[tier] / 16;
    for (int i = tid; i < n16; i += blockDim.x) p4[i] = make_uint4(0, 0, 0, 0);
  }
  __syncthreads();

  if (tier == KVQ_TIER_16) {
    if (tid < D) {
#pragma unroll
      for (int kind = 0; kind < 2; ++kind) {
        int w, bit;
        elem_pos(kind, 0, D, t, tid, w, bit);
        reinterpret_cast<uint16_t*>(chunk[kind])[2 * w + (bit >> 4)] = xb[kind][tid];
      }
    }
  } else {
    const int warp = tid >> 5, lane = tid & 31;
    const int ng = D / kGroup;
    for (int gi = warp; gi < 2 * ng; gi += 4) {
      const int kind = gi / ng, grp = gi % ng, d = grp * kGroup + lane;
      const QOut q = quant_group(xs[kind][d], tier, ov);
      codes[kind][d] = q.code;
      if (lane == 0) metas[kind][grp] = q.meta;
    }
    __syncthreads();
    const int b_bits = tier_bits(tier);
    if (tid < D) {
#pragma unroll
      for (int kind = 0; kind < 2; ++kind) {
        int w, bit;
        elem_pos(kind, tier, D, t, tid, w, bit);
        uint32_t* word = reinterpret_cast<uint32_t*>(chunk[kind]) + w;
        const uint32_t mask = ((1u << b_bits) - 1u) << bit;
        atomicAnd(word, ~mask);
        atomicOr(word, codes[kind][tid] << bit);
      }
    }
    if (tid < 2 * ng) {
      const int kind = tid / ng, grp = tid % ng;
      unsigned char* meta = chunk[kind] + codes_bytes(tier, D);
      if (tier == KVQ_TIER_I1)
        reinterpret_cast<uint16_t*>(meta)[t * ng + grp] = static_cast<uint16_t>(metas[kind][grp]);
      else
        reinterpret_cast<uint32_t*>(meta)[t * ng + grp] = metas[kind][grp];
    }
  }
  if (ov) set_err(c.err, KVQ_DERR_FP16_RANGE);
  if (nonfinite) set_err(c.err, KVQ_DERR_NONFINITE);
  griddep_launch_dependents();
}

// ----------------------------------------------------------------------------- build
template <bool BF16>
__global__ void __launch_bounds__(128) build_kernel(DevCache c, const uint16_t* __restrict__ ksrc,
                                                    const uint16_t* __restrict__ vsrc,
                                                    const int64_t* __restrict__ cu, int64_t src_tokens) {
  const int p = blockIdx.x;
  const int bg = blockIdx.y;
  const int b = bg / c.Hkv, g = bg % c.Hkv;
  const int D = c.D;
  const int tid = threadIdx.x;
  const int L = c.seq_len[b];
  const int P = (L + kPage - 1) / kPage;
  if (p >= P || p >= c.max_pages) return;
  const int n = min(kPage, L - p * kPage);
  const int64_t row0 = cu[b] + (int64_t)p * kPage;
  if (row0 < 0 || row0 + n > src_tokens) {
    if (tid == 0) set_err(c.err, KVQ_DERR_BAD_POS);
    return;
  }
  int tier;
  const unsigned char* ck;
  if (!page_chunk(c, b, p, g, tier, ck)) return;
  unsigned char* out = const_cast<unsigned char*>(ck);
  const int CB = c.chunk[tier];

  __shared__ __align__(16) uint32_t words[2][1024];  // chunk images (<= 4 KB each at D <= 128)
  __shared__ uint16_t xb[2][kPage][128];
  bool ov = false, nonfinite = false;

  for (int i = tid; i < 2 * 1024; i += blockDim.x) (&words[0][0])[i] = 0u;
  for (int i = tid; i < n * D; i += blockDim.x) {
    const int t = i / D, d = i % D;
    const size_t src = ((size_t)g * src_tokens + (size_t)(row0 + t)) * D + d;
    xb[0][t][d] = ksrc[src];
    xb[1][t][d] = vsrc[src];
  }
  __syncthreads();

  if (tid < D) {  // summary: fp64 sum of the page's keys in token order
    double S = 0.0;
    for (int t = 0; t < n; ++t) S += to_double<BF16>(xb[0][t][tid]);
    c.summary[((size_t)bg * c.max_pages + p) * D + tid] = fp16_sat(S / static_cast<double>(n), ov);
    if (p == P - 1) c.open_ksum[(size_t)bg * D + tid] = (L % kPage) ? S : 0.0;
  }

  if (tier == KVQ_TIER_16) {
    for (int e = tid; e < 2 * n * D; e += blockDim.x) {
      const int kind = e / (n * D), rem = e % (n * D), t = rem / D, d = rem % D;
      int w, bit;
      elem_pos(kind, 0, D, t, d, w, bit);
      reinterpret_cast<uint16_t*>(words[kind])[2 * w + (bit >> 4)] = xb[kind][t][d];
    }
  } else {
    const int warp = tid >> 5, lane = tid & 31;
    const int ng = D / kGroup;
    const int groups = 2 * n * ng;
    for (int gi = warp; gi < groups; gi += 4) {
      const int kind = gi / (n * ng), rem = gi % (n * ng), t = rem / ng, grp = rem % ng;
      const int d = grp * kGroup + lane;
      const double x = to_double<BF16>(xb[kind][t][d]);
      nonfinite |= !isfinite(x);
      const QOut q = quant_group(x, tier, ov);
      int w, bit;
      elem_pos(kind, tier, D, t, d, w, bit);
      atomicOr(&words[kind][w], q.code << bit);
      if (lane == 0) {
        unsigned char* meta = reinterpret_cast<unsigned char*>(words[kind]) + codes_bytes(tier, D);
        if (tier == KVQ_TIER_I1)
          reinterpret_cast<uint16_t*>(meta)[t * ng + grp] = static_cast<uint16_t>(q.meta);
        else
          reinterpret_cast<uint32_t*>(meta)[t * ng + grp] = q.meta;
      }
    }
  }
  __syncthreads();
  for (int kind = 0; kind < 2; ++kind) {
    const uint4* src = reinterpret_cast<const uint4*>(words[kind]);
    uint4* dst = reinterpret_cast<uint4*>(out + (size_t)kind * CB);
    for (int i = tid; i < CB / 16; i += blockDim.x) dst[i] = src[i];
  }
  if (ov) set_err(c.err, KVQ_DERR_FP16_RANGE);
  if (nonfinite) set_err(c.err, KVQ_DERR_NONFINITE);
}

}  // namespace

cudaError_t launch_append(const DevCache& c, const int32_t* pos, const void* k_new, const void* v_new,
                          cudaStream_t s) {
  const dim3 grid(c.B * c.Hkv);
  const uint16_t* kn = static_cast<const uint16_t*>(k_new);
  const uint16_t* vn = static_cast<const uint16_t*>(v_new);
  if (c.dtype == KVQ_DT_BF16) return launch_pdl(append_kernel<true>, grid, dim3(128), 0, s, c, pos, kn, vn);
  return launch_pdl(append_kernel<false>, grid, dim3(128), 0, s, c, pos, kn, vn);
}

cudaError_t launch_build(const DevCache& c, const void* k_src, const void* v_src, const int64_t* cu,
                         int64_t src_tokens, cudaStream_t s) {
  const dim3 grid(c.max_pages, c.B * c.Hkv);
  if (c.dtype == KVQ_DT_BF16)
    build_kernel<true><<<grid, 128, 0, s>>>(c, static_cast<const uint16_t*>(k_src),
                                            static_cast<const uint16_t*>(v_src), cu, src_tokens);
  else
    build_kernel<false><<<grid, 128, 0, s>>>(c, static_cast<const uint16_t*>(k_src),
                                             static_cast<const uint16_t*>(v_src), cu, src_tokens);
  return cudaGetLastError();
}

}  // namespace kvq
