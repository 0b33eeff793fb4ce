// Quantise-and-pack: kvq_append (one token per sequence), kvq_build_pages (whole pages) and
// kvq_requantize_pages (tier demotion of whole pages).
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
#include <utility>

#include "kvq_internal.cuh"
#include "quant.cuh"

namespace kvq {
namespace {

// ----------------------------------------------------------------------------- append
// One CTA of four warps per (b, kv head): the summary and the page clear over all 128
// threads, then one (kind, group) pair per warp at D = 128.
template <bool BF16>
__global__ void __launch_bounds__(128) append_kernel(DevCache c, const int32_t* __restrict__ pos,
                                                     const uint16_t* __restrict__ k_new,
                                                     const uint16_t* __restrict__ v_new) {
  __shared__ uint16_t s_k[128], s_v[128];  // the token's K and V rows (D <= 128)
  __shared__ double s_ks[128];              // the open page's fp64 key sums
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bg = blockIdx.x;
  const int b = bg / c.Hkv, g = bg % c.Hkv;
  // The page-score sweep that follows reads, before it waits for this grid, every summary
  // row except the ones this grid writes; it may launch as soon as everything before this
  // grid is complete, so that its sweep overlaps this kernel.
  griddep_wait();
  griddep_launch_dependents();
  // The rows and the sums do not depend on the page: fetched in the same round trip as
  // pos, ahead of the block-table lookup.
  const int P = pos[b];
  if (tid < c.D) {
    s_k[tid] = k_new[(size_t)bg * c.D + tid];
    s_v[tid] = v_new[(size_t)bg * c.D + tid];
    s_ks[tid] = c.open_ksum[(size_t)bg * c.D + tid];
  }
  __syncthreads();
  if (P >= c.max_pages * kPage) {
    if (tid == 0) set_err(c.err, KVQ_DERR_BAD_POS);
  } else if (P >= 0) {
    const bool ok = append_phase1<BF16>(c, b, g, P, s_k, tid, 128, nullptr, s_ks);
    __syncthreads();
    if (ok) append_phase2<BF16>(c, b, g, P, s_k, s_v, warp, 4, lane);
  }
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
  const unsigned char *ck, *cv;
  if (!page_chunks(c, b, p, g, tier, ck, cv)) return;
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
        if (tier == KVQ_TIER_I1 || tier == KVQ_TIER_F8)
          reinterpret_cast<uint16_t*>(meta)[t * ng + grp] = static_cast<uint16_t>(q.meta);
        else
          reinterpret_cast<uint32_t*>(meta)[t * ng + grp] = q.meta;
      }
    }
  }
  __syncthreads();
  for (int kind = 0; kind < 2; ++kind) {
    const uint4* src = reinterpret_cast<const uint4*>(words[kind]);
    uint4* dst = reinterpret_cast<uint4*>(const_cast<unsigned char*>(kind ? cv : ck));
    for (int i = tid; i < CB / 16; i += blockDim.x) dst[i] = src[i];
  }
  if (ov) set_err(c.err, KVQ_DERR_FP16_RANGE);
  if (nonfinite) set_err(c.err, KVQ_DERR_NONFINITE);
}

// Tier demotion (ARGUS "Virtual Memory for Transformers", "Visual Architecture": pages
// move down the cascade of tiers as they cool).  Item i = (b, page, new entry): the page's
// tokens are read back from their current tier and quantised again, per token and
// 32-channel group, into the new entry's b-bit tier and slot; a second launch then points
// the block table at the new slot.  Both launches decide an item's validity the same way,
// from a block table that only the second one changes: b and page in range, the page
// holds tokens, the current entry is valid, and the new entry is a b-bit tier slot other
// than the current one.
__device__ inline bool requant_item(const DevCache& c, const int32_t* items, int i, int& b, int& p, uint32_t& oe,
                                    uint32_t& ne, int& n) {
  b = items[3 * i];
  p = items[3 * i + 1];
  ne = static_cast<uint32_t>(items[3 * i + 2]);
  if (b < 0 || b >= c.B || p < 0 || p >= c.max_pages) return false;
  n = min(kPage, c.seq_len[b] - p * kPage);
  if (n <= 0) return false;
  oe = static_cast<uint32_t>(c.block_table[(size_t)b * c.max_pages + p]);
  const int ot = static_cast<int>(oe >> 29), nt = static_cast<int>(ne >> 29);
  const long long os = oe & 0x1FFFFFFFu, ns = ne & 0x1FFFFFFFu;
  if (ot >= kNumTiers || c.pool[ot] == nullptr || os >= c.pool_slots[ot]) return false;
  if (nt < 1 || nt >= kNumTiers || c.pool[nt] == nullptr || ns >= c.pool_slots[nt]) return false;
  return !(nt == ot && ns == os);
}

// Re-quantiser of one (page, kv head), 128 threads, in three phases over shared memory:
//  A  decode the current chunk word by word into fp32 values vals[j][group], group =
//     (kind * 16 + t) * (D / 32) + d / 32 and j = d % 32 (one row per channel of a group,
//     so that phase B reads without bank conflicts);
//  B  one thread per (kind, token, 32-channel group): the group's min and max, its fp16
//     zero and scale in fp64 as quant_group computes them, then each code from an fp32
//     quotient; a quotient within 1e-4 of a rounding tie (or not finite) is recomputed
//     exactly in fp64.  Away from ties both round to the same integer: the fp32 quotient
//     is within 3 * 2^-24 relative of the exact one, i.e. within 5e-5 where the clamp to
//     [0, 2^b - 1] does not decide the code.  Code bytes go to shared memory, metadata
//     straight to the new chunk;
//  C  one thread per word of the new codes area gathers its codes: one store per word.
constexpr int kRqGroups = 2 * kPage * 128 / kGroup;  // groups per (page, kv head), D <= 128

template <int OT, int KIND, int D, bool BF16, bool FULL, int I>
__device__ inline void rq_decode_word(const uint32_t* chunk, int W0, int n, float (*vals)[kRqGroups + 1]) {
  constexpr int ng = D / kGroup;
  const unsigned char* meta = reinterpret_cast<const unsigned char*>(chunk) + codes_bytes(OT, D);
  const uint32_t word = chunk[W0 + 128 * I];
  word_elems_at<OT, KIND, D, I>(W0, [&](int t, int d, int sh) {
    if (!FULL && t >= n) return;
    float v;
    if constexpr (OT == KVQ_TIER_16) {
      v = bits_to_float<BF16>(static_cast<uint16_t>(word >> sh));
    } else {
      const uint32_t code = (word >> sh) & ((1u << tier_bits(OT)) - 1u);
      if constexpr (OT == KVQ_TIER_I1) {
        const float m = __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(meta)[t * ng + (d >> 5)]));
        v = code ? m : -m;
      } else if constexpr (OT == KVQ_TIER_F8) {
        v = e4m3_to_float(code) *
            __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(meta)[t * ng + (d >> 5)]));
      } else {
        const uint32_t mw = reinterpret_cast<const uint32_t*>(meta)[t * ng + (d >> 5)];
        v = fmaf(static_cast<float>(code), __half2float(__ushort_as_half(static_cast<uint16_t>(mw & 0xFFFFu))),
                 __half2float(__ushort_as_half(static_cast<uint16_t>(mw >> 16))));
      }
    }
    vals[d & 31][(KIND * kPage + t) * ng + (d >> 5)] = v;
  });
}

// Thread W0 (< 128) decodes words W0, W0 + 128, ... of the K then the V codes area.
template <int OT, int KIND, int D, bool BF16, bool FULL, int... Is>
__device__ inline void rq_decode_kind(const uint32_t* chunk, int n, float (*vals)[kRqGroups + 1],
                                      std::integer_sequence<int, Is...>) {
  constexpr int wpk = codes_bytes(OT, D) / 4;
  const int W0 = threadIdx.x;
  ((W0 + 128 * Is < wpk ? rq_decode_word<OT, KIND, D, BF16, FULL, Is>(chunk, W0, n, vals) : void()), ...);
}

template <int OT, int D, bool BF16>
__device__ inline void rq_decode(const uint32_t* oldw, int n, float (*vals)[kRqGroups + 1]) {
  constexpr int wpk = codes_bytes(OT, D) / 4, cw = chunk_bytes(OT, D) / 4;
  using Seq = std::make_integer_sequence<int, (wpk + 127) / 128>;
  if (n == kPage) {  // a full page: no token-range test per element
    rq_decode_kind<OT, 0, D, BF16, true>(oldw, n, vals, Seq{});
    rq_decode_kind<OT, 1, D, BF16, true>(oldw + cw, n, vals, Seq{});
  } else {
    rq_decode_kind<OT, 0, D, BF16, false>(oldw, n, vals, Seq{});
    rq_decode_kind<OT, 1, D, BF16, false>(oldw + cw, n, vals, Seq{});
  }
}

template <int NT, int D>
__device__ inline void rq_quant(int gid, int n, const float (*vals)[kRqGroups + 1], unsigned char* codes8,
                                unsigned char* dstK, unsigned char* dstV, bool& ov, bool& nonfinite) {
  constexpr int ng = D / kGroup;
  const int kind = gid / (kPage * ng), t = (gid / ng) % kPage, grp = gid % ng;
  uint4* crow = reinterpret_cast<uint4*>(codes8 + (kind * kPage + t) * D + grp * kGroup);
  unsigned char* meta = (kind ? dstV : dstK) + codes_bytes(NT, D);
  if (t >= n) {  // token slot past the sequence: zero codes and metadata
    crow[0] = crow[1] = make_uint4(0, 0, 0, 0);
    if constexpr (NT == KVQ_TIER_I1 || NT == KVQ_TIER_F8) reinterpret_cast<uint16_t*>(meta)[t * ng + grp] = 0;
    else reinterpret_cast<uint32_t*>(meta)[t * ng + grp] = 0u;
    return;
  }
  float v[kGroup];
#pragma unroll
  for (int j = 0; j < kGroup; ++j) v[j] = vals[j][gid];
  uint32_t packed[kGroup / 4];
  if constexpr (NT == KVQ_TIER_F8) {  // scale fp16(amax / 448), code e4m3(x / scale) from the fp64 quotient
    float amax = 0.0f;
    bool bad = false;
#pragma unroll
    for (int j = 0; j < kGroup; ++j) {
      amax = fmaxf(amax, fabsf(v[j]));
      bad |= !isfinite(v[j]);
    }
    // a group holding a non-finite value: NaN scale and zero codes (it reads back as NaN)
    const uint16_t sb = bad ? kF8NaNScale : fp16_sat(static_cast<double>(amax) / 448.0, ov);
    const double sc = bad ? 0.0 : static_cast<double>(__half2float(__ushort_as_half(sb)));
#pragma unroll
    for (int k = 0; k < kGroup / 4; ++k) {
      packed[k] = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float x = v[4 * k + i];
        nonfinite |= !isfinite(x);
        const uint32_t code =
            sc != 0.0 ? __nv_cvt_double_to_fp8(static_cast<double>(x) / sc, __NV_SATFINITE, __NV_E4M3) : 0u;
        packed[k] |= code << (8 * i);
      }
    }
    reinterpret_cast<uint16_t*>(meta)[t * ng + grp] = sb;
  } else if constexpr (NT == KVQ_TIER_I1) {
    double s = 0.0;
#pragma unroll
    for (int j = 0; j < kGroup; ++j) s += fabs(static_cast<double>(v[j]));
    nonfinite |= !isfinite(s);  // an infinite or NaN value makes the sum so
#pragma unroll
    for (int k = 0; k < kGroup / 4; ++k) {
      packed[k] = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) packed[k] |= (v[4 * k + i] >= 0.0f ? 1u : 0u) << (8 * i);
    }
    reinterpret_cast<uint16_t*>(meta)[t * ng + grp] = fp16_sat(s / 32.0, ov);
  } else {
    constexpr int qmax = (1 << tier_bits(NT)) - 1;
    float lo = v[0], hi = v[0];
#pragma unroll
    for (int j = 0; j < kGroup; ++j) {
      lo = fminf(lo, v[j]);
      hi = fmaxf(hi, v[j]);
    }
    const double lod = static_cast<double>(lo) + 0.0, hid = static_cast<double>(hi) + 0.0;
    const uint16_t zb = fp16_sat(lod, ov);
    const uint16_t sb = fp16_sat((hid - lod) / static_cast<double>(qmax), ov);
    const float zf = __half2float(__ushort_as_half(zb)), sf = __half2float(__ushort_as_half(sb));
    const float inv = 1.0f / sf;
    if (sf == 0.0f) {  // constant group (min/max skip NaN: check the values)
#pragma unroll
      for (int j = 0; j < kGroup; ++j) nonfinite |= !isfinite(v[j]);
#pragma unroll
      for (int k = 0; k < kGroup / 4; ++k) packed[k] = 0;
    } else {
#pragma unroll
      for (int k = 0; k < kGroup / 4; ++k) {
        packed[k] = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float x = v[4 * k + i];
          const float q = (x - zf) * inv;
          float c = rintf(q);
          if (!(fabsf(q - c) < 0.4999f)) {  // near a tie, or not finite (every non-finite x lands here)
            nonfinite |= !isfinite(x);
            c = static_cast<float>(
                rint((static_cast<double>(x) - static_cast<double>(zf)) / static_cast<double>(sf)));
          }
          // clamp to [0, qmax] (fmaxf maps NaN to 0); the codes of a word do not overlap
          packed[k] += min(__float2uint_rn(fmaxf(c, 0.0f)), static_cast<uint32_t>(qmax)) << (8 * i);
        }
      }
    }
    reinterpret_cast<uint32_t*>(meta)[t * ng + grp] = static_cast<uint32_t>(sb) | (static_cast<uint32_t>(zb) << 16);
  }
  crow[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  crow[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
}

template <int NT, int KIND, int D, int I>
__device__ inline void rq_pack_word(const unsigned char* codes8, uint32_t* d32, int W0) {
  uint32_t acc = 0;
  word_elems_at<NT, KIND, D, I>(W0, [&](int t, int d, int sh) { acc |= static_cast<uint32_t>(codes8[t * D + d]) << sh; });
  d32[W0 + 128 * I] = acc;
}

template <int NT, int KIND, int D, int... Is>
__device__ inline void rq_pack_kind(const unsigned char* codes8, uint32_t* d32, std::integer_sequence<int, Is...>) {
  constexpr int wpk = codes_bytes(NT, D) / 4;
  const int W0 = threadIdx.x;
  ((W0 + 128 * Is < wpk ? rq_pack_word<NT, KIND, D, Is>(codes8, d32, W0) : void()), ...);
}

template <int NT, int D>
__device__ inline void rq_pack(const unsigned char* codes8, unsigned char* dstK, unsigned char* dstV) {
  constexpr int wpk = codes_bytes(NT, D) / 4;
  using Seq = std::make_integer_sequence<int, (wpk + 127) / 128>;
  rq_pack_kind<NT, 0, D>(codes8, reinterpret_cast<uint32_t*>(dstK), Seq{});
  rq_pack_kind<NT, 1, D>(codes8 + kPage * D, reinterpret_cast<uint32_t*>(dstV), Seq{});
}

template <bool BF16, int D>
__global__ void __launch_bounds__(128) requant_kernel(DevCache c, const int32_t* __restrict__ items) {
  const int g = blockIdx.y, tid = threadIdx.x;
  int b, p, n;
  uint32_t oe, ne;
  if (!requant_item(c, items, blockIdx.x, b, p, oe, ne, n)) {
    if (g == 0 && tid == 0) set_err(c.err, KVQ_DERR_BAD_PAGE);
    return;
  }
  const int ot = static_cast<int>(oe >> 29), nt = static_cast<int>(ne >> 29);
  const int OB = chunk_bytes(ot, D), NB = chunk_bytes(nt, D);
  const unsigned char *srcK, *srcV, *dK, *dV;
  slot_chunks(c, ot, oe & 0x1FFFFFFFu, g, srcK, srcV);
  slot_chunks(c, nt, ne & 0x1FFFFFFFu, g, dK, dV);
  unsigned char* dstK = const_cast<unsigned char*>(dK);
  unsigned char* dstV = const_cast<unsigned char*>(dV);

  __shared__ __align__(16) uint32_t old_words[2 * chunk_bytes(KVQ_TIER_16, 128) / 4];
  __shared__ float vals[kGroup][kRqGroups + 1];
  __shared__ __align__(16) unsigned char codes8[2 * kPage * 128];
  for (int k = tid; k < 2 * OB / 16; k += blockDim.x)
    reinterpret_cast<uint4*>(old_words)[k] =
        __ldcg(k < OB / 16 ? reinterpret_cast<const uint4*>(srcK) + k : reinterpret_cast<const uint4*>(srcV) + (k - OB / 16));
  __syncthreads();
  switch (ot) {
    case 0: rq_decode<0, D, BF16>(old_words, n, vals); break;
    case 1: rq_decode<1, D, BF16>(old_words, n, vals); break;
    case 2: rq_decode<2, D, BF16>(old_words, n, vals); break;
    case 3: rq_decode<3, D, BF16>(old_words, n, vals); break;
    case 4: rq_decode<4, D, BF16>(old_words, n, vals); break;
    default: rq_decode<5, D, BF16>(old_words, n, vals); break;
  }
  __syncthreads();
  bool ov = false, nonfinite = false;
  if (tid < 2 * kPage * (D / kGroup)) {
    switch (nt) {
      case 1: rq_quant<1, D>(tid, n, vals, codes8, dstK, dstV, ov, nonfinite); break;
      case 2: rq_quant<2, D>(tid, n, vals, codes8, dstK, dstV, ov, nonfinite); break;
      case 3: rq_quant<3, D>(tid, n, vals, codes8, dstK, dstV, ov, nonfinite); break;
      case 4: rq_quant<4, D>(tid, n, vals, codes8, dstK, dstV, ov, nonfinite); break;
      default: rq_quant<5, D>(tid, n, vals, codes8, dstK, dstV, ov, nonfinite); break;
    }
  }
  __syncthreads();
  switch (nt) {
    case 1: rq_pack<1, D>(codes8, dstK, dstV); break;
    case 2: rq_pack<2, D>(codes8, dstK, dstV); break;
    case 3: rq_pack<3, D>(codes8, dstK, dstV); break;
    case 4: rq_pack<4, D>(codes8, dstK, dstV); break;
    default: rq_pack<5, D>(codes8, dstK, dstV); break;
  }
  if (ov) set_err(c.err, KVQ_DERR_FP16_RANGE);
  if (nonfinite) set_err(c.err, KVQ_DERR_NONFINITE);
}

__global__ void requant_commit_kernel(DevCache c, const int32_t* __restrict__ items, int n_items) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_items) return;
  int b, p, n;
  uint32_t oe, ne;
  if (requant_item(c, items, i, b, p, oe, ne, n))
    const_cast<int32_t*>(c.block_table)[(size_t)b * c.max_pages + p] = static_cast<int32_t>(ne);
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

cudaError_t launch_requantize(const DevCache& c, const int32_t* items, int n, cudaStream_t s) {
  const dim3 grid(n, c.Hkv);
  const bool bf = c.dtype == KVQ_DT_BF16;
  if (c.D == 128) {
    if (bf) requant_kernel<true, 128><<<grid, 128, 0, s>>>(c, items);
    else requant_kernel<false, 128><<<grid, 128, 0, s>>>(c, items);
  } else {
    if (bf) requant_kernel<true, 64><<<grid, 128, 0, s>>>(c, items);
    else requant_kernel<false, 64><<<grid, 128, 0, s>>>(c, items);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  requant_commit_kernel<<<(n + 255) / 256, 256, 0, s>>>(c, items, n);
  return cudaGetLastError();
}

}  // namespace kvq
