// Per-group quantiser of one token (warp-collective, IEEE binary64, round-half-even) and
// the one-warp token append built on it, shared by the append, the page builder and the
// fused decode step.
//
// ARGUS "Virtual Memory for Transformers", "Visual Architecture": INT8 / INT4 / INT2 /
// 1-bit cold tiers (and FP8 e4m3: scale = fp16(max|x| / 448), code = e4m3(x / scale)
// rounded half to even with saturation).  Per 32-channel group: zero = fp16(min), scale =
// fp16((max - min) / (2^b - 1)), code = clamp(rint((x - zero) / scale), 0, 2^b - 1) (0 when
// scale == 0); 1-bit: sign (x >= 0) and magnitude fp16(sum|x| / 32) summed in channel order.
// Every step is an IEEE binary64 operation with round-half-even, so the bytes do not depend
// on the thread mapping.  The per-page mean-key summary (AMASS "What is in the box": a
// tiny per-page summary) is fp16(S / n) with S the fp64 sum of the page's keys in token
// order.
#pragma once

#include "kvq_internal.cuh"

namespace kvq {

struct QOut {
  uint32_t code;
  uint32_t meta;  // INT-b: scale | zero << 16 ; 1-bit: magnitude
};

// FP8 scale bits stored for a group that holds a non-finite value (an fp16 quiet NaN).
constexpr uint16_t kF8NaNScale = 0x7E00u;

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
  if (tier == KVQ_TIER_F8) {  // e4m3 with scale fp16(amax / 448), round-half-even, saturating
    double a = fabs(x);
#pragma unroll
    for (int o = 16; o; o >>= 1) a = fmax(a, __shfl_xor_sync(full, a, o));
    a += 0.0;
    const uint16_t sb = fp16_sat(a / 448.0, ov);
    // a group holding a non-finite value: NaN scale and zero codes, so it reads back as NaN
    if (__any_sync(full, !isfinite(x))) return {0u, kF8NaNScale};
    const double scale = static_cast<double>(__half2float(__ushort_as_half(sb)));
    const uint32_t code = scale != 0.0 ? __nv_cvt_double_to_fp8(x / scale, __NV_SATFINITE, __NV_E4M3) : 0u;
    return {code, sb};
  }
  double lo = x, hi = x;
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    lo = fmin(lo, __shfl_xor_sync(full, lo, o));
    hi = fmax(hi, __shfl_xor_sync(full, hi, o));
  }
  lo += 0.0;  // a zero extreme is +0, whichever zero the reduction met first
  hi += 0.0;
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

// Token append, in two phases so that several warps can share it (the caller puts a
// barrier over those warps between the phases):
//  phase 1 (threads t0 = 0 .. nt-1): advance the open page's fp64 key sum and its fp16
//          summary (`patch`, nullable, receives the new summary row too), and clear a newly
//          opened page;
//  phase 2 (warps w = 0 .. nw-1): quantise K and V into the page's tier, warp w taking the
//          (kind, 32-channel group) pairs w, w + nw, ...
// Token `pos` of sequence b, kv head g; the caller has checked 0 <= pos < max_pages * 16.
// Both phases return false (nothing written) if the page's block-table entry is invalid.
template <bool BF16>
__device__ inline bool append_phase1(const DevCache& c, int b, int g, int pos, const uint16_t* krow, int t0, int nt,
                                     uint16_t* patch, const double* ksum_src = nullptr) {
  const int D = c.D;
  const size_t bg = (size_t)b * c.Hkv + g;
  const int page = pos / kPage, t = pos % kPage;
  int tier;
  const unsigned char *ck, *cv;
  if (!page_chunks(c, b, page, g, tier, ck, cv)) return false;
  bool ov = false;
  for (int d = t0; d < D; d += nt) {  // running key sum of the open page and its summary
    const double x = to_double<BF16>(krow[d]);
    double* ks = c.open_ksum + bg * D + d;  // ksum_src: the same sums, already fetched
    const double S = (t == 0) ? x : ((ksum_src != nullptr ? ksum_src[d] : *ks) + x);
    *ks = S;
    const uint16_t m = fp16_sat(S / static_cast<double>(t + 1), ov);
    c.summary[(bg * c.max_pages + page) * D + d] = m;
    if (patch != nullptr) patch[d] = m;
  }
  if (ov) set_err(c.err, KVQ_DERR_FP16_RANGE);
  if (t == 0) {  // a newly opened page starts from zero bytes
    uint4* k4 = reinterpret_cast<uint4*>(const_cast<unsigned char*>(ck));
    uint4* v4 = reinterpret_cast<uint4*>(const_cast<unsigned char*>(cv));
    const int n16 = c.chunk[tier] / 16;
    for (int i = t0; i < 2 * n16; i += nt) (i < n16 ? k4[i] : v4[i - n16]) = make_uint4(0, 0, 0, 0);
  }
  return true;
}

template <bool BF16>
__device__ inline bool append_phase2(const DevCache& c, int b, int g, int pos, const uint16_t* krow,
                                     const uint16_t* vrow, int w, int nw, int lane) {
  const int D = c.D;
  const int page = pos / kPage, t = pos % kPage;
  int tier;
  const unsigned char *ck, *cv;
  if (!page_chunks(c, b, page, g, tier, ck, cv)) return false;
  bool ov = false, nonfinite = false;
  const int ng = D / kGroup;
  for (int gi = w; gi < 2 * ng; gi += nw) {
    const int kind = gi / ng, grp = gi % ng;
    const int d = grp * kGroup + lane;
    unsigned char* chunk = const_cast<unsigned char*>(kind ? cv : ck);
    const uint16_t v = (kind ? vrow : krow)[d];
    const double x = to_double<BF16>(v);
    nonfinite |= !isfinite(x);
    int wd, bit;
    elem_pos(kind, tier, D, t, d, wd, bit);
    if (tier == KVQ_TIER_16) {
      reinterpret_cast<uint16_t*>(chunk)[2 * wd + (bit >> 4)] = v;
      continue;
    }
    const QOut q = quant_group(x, tier, ov);
    const uint32_t cmask = (1u << tier_bits(tier)) - 1u;
    uint32_t* word = reinterpret_cast<uint32_t*>(chunk) + wd;
    atomicAnd(word, ~(cmask << bit));  // lanes of one group can share a word
    atomicOr(word, q.code << bit);
    if (lane == 0) {
      unsigned char* meta = chunk + codes_bytes(tier, D);
      if (tier == KVQ_TIER_I1 || tier == KVQ_TIER_F8)
        reinterpret_cast<uint16_t*>(meta)[t * ng + grp] = static_cast<uint16_t>(q.meta);
      else
        reinterpret_cast<uint32_t*>(meta)[t * ng + grp] = q.meta;
    }
  }
  if (__any_sync(0xffffffffu, ov) && lane == 0) set_err(c.err, KVQ_DERR_FP16_RANGE);
  if (__any_sync(0xffffffffu, nonfinite) && lane == 0) set_err(c.err, KVQ_DERR_NONFINITE);
  return true;
}

// One warp does both phases.
template <bool BF16>
__device__ inline bool append_token_warp(const DevCache& c, int b, int g, int pos, const uint16_t* krow,
                                         const uint16_t* vrow, int lane, uint16_t* patch) {
  const bool ok = append_phase1<BF16>(c, b, g, pos, krow, lane, 32, patch);
  __syncwarp();
  return ok && append_phase2<BF16>(c, b, g, pos, krow, vrow, 0, 1, lane);
}

}  // namespace kvq
