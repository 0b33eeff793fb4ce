// Per-page attention math shared by the sparse decode attention and the fused decode
// step: one warp, one page of 16 tokens, the kv head's G <= 8 query heads.
//
// Warp-level tensor-core mma m16n8k16 with fp32 accumulation:
//   S^T[t][h] = K[t][:] . q[h][:]      A = K rows (tokens), B = q^T (heads as N)
//   O^T[d][h] += V^T[d][:] . P^T[:][h] A = V^T rows (channels), B = P^T via movmatrix
// The page byte order is the mma operand order, so every operand is one 16-byte
// conflict-free shared-memory load per lane.  Quantised pages: codes are converted
// exactly to centred 16-bit floats c - 2^(b-1) in registers (magic-exponent bit tricks)
// and the per-group affine map is applied around the mma with z' = zero + 2^(b-1)*scale:
// for K, S += scale_t * (codes . q) + z'_t * sum(q over the group); for V, P^T is scaled
// per token by the group's scale before the mma and sum_t z'_t * p_t is accumulated on
// the side.  FP8 (e4m3) pages convert their codes exactly to fp16 / bf16 and have no zero
// offset (S += scale_t * (codes . q); V: P^T scaled per token).  P^T enters the tensor core as a 16-bit hi + lo pair (two mmas), so the only
// 16-bit rounding on the way to the output is the final cast.  Online softmax runs in
// the log2 domain.
#pragma once

#include <math.h>

#include "kvq_internal.cuh"
#include "ptx.cuh"

namespace kvq {

template <bool BF16>
__device__ inline uint32_t pack2(float lo, float hi) {
  if constexpr (BF16) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
  } else {
    const __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
  }
}
// (hi, lo) 16-bit pairs with hi + lo = (a, b) to ~2^-17 relative: the P^T operand
// is fed to the tensor core as two terms so its 16-bit rounding does not reach the output.
template <bool BF16>
__device__ inline void split2(float a, float b, uint32_t& hi, uint32_t& lo) {
  hi = pack2<BF16>(a, b);
  float ah, bh;
  if constexpr (BF16) {
    ah = __uint_as_float(hi << 16);
    bh = __uint_as_float(hi & 0xFFFF0000u);
  } else {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hi));
    ah = f.x;
    bh = f.y;
  }
  lo = pack2<BF16>(a - ah, b - bh);
}
__device__ inline uint32_t sub2(uint32_t x, uint32_t y, bool bf16) {
  if (bf16) {
    const __nv_bfloat162 r = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&x),
                                     *reinterpret_cast<const __nv_bfloat162*>(&y));
    return *reinterpret_cast<const uint32_t*>(&r);
  }
  const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&x), *reinterpret_cast<const __half2*>(&y));
  return *reinterpret_cast<const uint32_t*>(&r);
}

// Exact 16-bit float pair (low, high) of the centred codes c - 2^(b-1) of register pair
// j of lane word w (1-bit: +-1).  Centring keeps the tensor-core term and the separate
// zero term small, so the 16-bit rounding of the other operand is not amplified by
// cancellation between them.
// FP8 e4m3 byte -> fp32, exact: the byte's exponent and mantissa placed in an fp32
// pattern, then scaled by 2^(127 - 7); e4m3 subnormals land on fp32 subnormals, so the
// product is exact for them too (NaN codes, from non-finite input, come out as 480).
__device__ inline float e4m3_bits_to_f32(uint32_t b) {
  return __uint_as_float(((b & 0x80u) << 24) | ((b & 0x7Fu) << 20)) * 0x1p120f;
}

template <int TIER, bool BF16>
__device__ inline uint32_t code_pair(uint32_t w, int j) {
  if constexpr (TIER == KVQ_TIER_F8) {  // e4m3 bytes j and j + 2: exact in fp16 and bf16
    if constexpr (BF16) {
      return pack2<true>(e4m3_bits_to_f32(w >> (8 * j)), e4m3_bits_to_f32(w >> (16 + 8 * j)));
    } else {
      const uint32_t x2 = __byte_perm(w, 0u, static_cast<uint32_t>(j | ((j + 2) << 4) | 0x4400));
      const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(x2), __NV_E4M3);
      return static_cast<uint32_t>(h.x) | (static_cast<uint32_t>(h.y) << 16);
    }
  } else if constexpr (TIER == KVQ_TIER_I1) {
    const uint32_t neg1 = BF16 ? 0xBF80BF80u : 0xBC00BC00u;  // (-1, -1)
    return ((w << (15 - j)) & 0x80008000u) ^ neg1;              // bit set -> +1
  } else if constexpr (TIER == KVQ_TIER_I8 && BF16) {
    // 2^23 + c as a float; subtracting 2^23 + 128 leaves c - 128, exact in bf16
    const float lo = __uint_as_float(0x4B000000u | ((w >> (8 * j)) & 0xFFu)) - 8388736.0f;
    const float hi = __uint_as_float(0x4B000000u | ((w >> (16 + 8 * j)) & 0xFFu)) - 8388736.0f;
    return pack2<true>(lo, hi);
  } else {
    constexpr int b = TIER == KVQ_TIER_I8 ? 8 : TIER == KVQ_TIER_I4 ? 4 : 2;
    constexpr uint32_t mask = ((1u << b) - 1u) * 0x00010001u;
    // 16-bit float with the exponent of 128 (bf16) / 1024 (fp16): mantissa units of 1
    constexpr uint32_t magic = BF16 ? 0x43004300u : 0x64006400u;
    constexpr uint32_t centre = magic | ((1u << (b - 1)) * 0x00010001u);
    return sub2(((w >> (b * j)) & mask) | magic, centre, BF16);
  }
}

// Lane words of a b-bit codes area (NW words per lane, stored in pieces of PW words).
template <int TIER, int D>
struct LaneWords {
  static constexpr int b = (TIER == KVQ_TIER_I8 || TIER == KVQ_TIER_F8) ? 8 : TIER == KVQ_TIER_I4 ? 4
                           : TIER == KVQ_TIER_I2 ? 2 : 1;
  static constexpr int NW = D * b / 64;
  static constexpr int PW = NW < 4 ? NW : 4;
  static constexpr int PPW = 16 / b;  // register pairs per word
  uint32_t w[NW];
  __device__ inline void load(const unsigned char* base, int lane) {
    const uint32_t* p = reinterpret_cast<const uint32_t*>(base);
#pragma unroll
    for (int pc = 0; pc < NW / PW; ++pc) {
      const uint32_t* src = p + ((size_t)pc * 32 + lane) * PW;
      if constexpr (PW == 4) {
        const uint4 v = *reinterpret_cast<const uint4*>(src);
        w[pc * 4 + 0] = v.x; w[pc * 4 + 1] = v.y; w[pc * 4 + 2] = v.z; w[pc * 4 + 3] = v.w;
      } else if constexpr (PW == 2) {
        const uint2 v = *reinterpret_cast<const uint2*>(src);
        w[pc * 2 + 0] = v.x; w[pc * 2 + 1] = v.y;
      } else {
        w[pc] = *src;
      }
    }
  }
  template <bool BF16>
  __device__ inline void frag(int kk, uint32_t (&a)[4]) const {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int R = 4 * kk + r;
      a[r] = code_pair<TIER, BF16>(w[R / PPW], R % PPW);
    }
  }
};

// N consecutive words with one vector load (src aligned to 4 * N bytes).
template <int N>
__device__ __forceinline__ void load_words(const uint32_t* src, uint32_t (&w)[N]) {
  if constexpr (N == 4) {
    const uint4 v = *reinterpret_cast<const uint4*>(src);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if constexpr (N == 2) {
    const uint2 v = *reinterpret_cast<const uint2*>(src);
    w[0] = v.x; w[1] = v.y;
  } else {
#pragma unroll
    for (int i = 0; i < N; ++i) w[i] = src[i];
  }
}

// Per-token metadata of one chunk for the lane's two token rows t0 = g8, t1 = g8 + 8:
// the scale s and the zero offset of the centred codes, z + 2^(b-1) * s (1-bit: m, 0;
// FP8: the scale, 0).  A token's NG metadata words (or half-words) are contiguous, and
// aligned to their total size (the metadata area of every chunk is 16-byte aligned), so
// they are read with one vector load.
template <int TIER, int D>
__device__ __forceinline__ void load_meta(const unsigned char* meta, int t0, float (&s)[2][D / 32],
                                          float (&z)[2][D / 32]) {
  constexpr int NG = D / 32;
  constexpr float half = TIER == KVQ_TIER_I8 ? 128.f : TIER == KVQ_TIER_I4 ? 8.f : 2.f;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int t = t0 + 8 * i;
    if constexpr (TIER == KVQ_TIER_I1 || TIER == KVQ_TIER_F8) {  // NG fp16 values per token
      uint32_t w[NG / 2];
      load_words<NG / 2>(reinterpret_cast<const uint32_t*>(meta) + t * (NG / 2), w);
#pragma unroll
      for (int gi = 0; gi < NG; ++gi) {
        s[i][gi] = __half2float(__ushort_as_half(static_cast<uint16_t>(w[gi / 2] >> (16 * (gi & 1)))));
        z[i][gi] = 0.f;
      }
    } else {
      uint32_t m[NG];
      load_words<NG>(reinterpret_cast<const uint32_t*>(meta) + t * NG, m);
#pragma unroll
      for (int gi = 0; gi < NG; ++gi) {
        const uint32_t v = m[gi];
        const float sc = __half2float(__ushort_as_half(static_cast<uint16_t>(v & 0xFFFFu)));
        s[i][gi] = sc;
        z[i][gi] = fmaf(half, sc, __half2float(__ushort_as_half(static_cast<uint16_t>(v >> 16))));
      }
    }
  }
}

template <int D>
struct WarpState {
  static constexpr int KS = D / 16;
  static constexpr int NG = D / 32;
  float m[2], l[2];
  float o[KS][4];
  float zacc[NG][2];
  uint32_t qb[KS][2];
  float qs[NG][2];
};

// S^T accumulation for one page: sacc = (t0,h0), (t0,h1), (t1,h0), (t1,h1)
template <int TIER, int D, bool BF16>
__device__ __forceinline__ void qk_page(const unsigned char* base, int lane, const WarpState<D>& st, float (&sacc)[4]) {
  constexpr int KS = D / 16, NG = D / 32;
  if constexpr (TIER == KVQ_TIER_16) {
    float s2[4] = {0.f, 0.f, 0.f, 0.f};  // second chain: halves the dependent-mma latency
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      const uint4 v = *reinterpret_cast<const uint4*>(base + ((size_t)kk * 32 + lane) * 16);
      const uint32_t a[4] = {v.x, v.y, v.z, v.w};
      if (kk & 1) mma16816<BF16>(s2, a, st.qb[kk][0], st.qb[kk][1]);
      else mma16816<BF16>(sacc, a, st.qb[kk][0], st.qb[kk][1]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) sacc[i] += s2[i];
  } else {
    LaneWords<TIER, D> lw;
    lw.load(base, lane);
    float s[2][NG], z[2][NG];
    load_meta<TIER, D>(base + codes_bytes(TIER, D), lane >> 2, s, z);
#pragma unroll
    for (int gi = 0; gi < NG; ++gi) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t a[4];
        lw.template frag<BF16>(2 * gi + h, a);
        mma16816<BF16>(acc, a, st.qb[2 * gi + h][0], st.qb[2 * gi + h][1]);
      }
      if constexpr (TIER == KVQ_TIER_F8) {  // no zero offset
        sacc[0] += s[0][gi] * acc[0];
        sacc[1] += s[0][gi] * acc[1];
        sacc[2] += s[1][gi] * acc[2];
        sacc[3] += s[1][gi] * acc[3];
      } else {
        sacc[0] += s[0][gi] * acc[0] + z[0][gi] * st.qs[gi][0];
        sacc[1] += s[0][gi] * acc[1] + z[0][gi] * st.qs[gi][1];
        sacc[2] += s[1][gi] * acc[2] + z[1][gi] * st.qs[gi][0];
        sacc[3] += s[1][gi] * acc[3] + z[1][gi] * st.qs[gi][1];
      }
    }
  }
}

// O^T += V^T P^T for one page; p = (t0,h0), (t0,h1), (t1,h0), (t1,h1)
template <int TIER, int D, bool BF16>
__device__ __forceinline__ void pv_page(const unsigned char* base, int lane, WarpState<D>& st, const float (&p)[4]) {
  constexpr int KS = D / 16, NG = D / 32;
  if constexpr (TIER == KVQ_TIER_16) {
    uint32_t h0, l0, h1, l1;
    split2<BF16>(p[0], p[1], h0, l0);
    split2<BF16>(p[2], p[3], h1, l1);
    const uint32_t b0h = movmatrix_t(h0), b1h = movmatrix_t(h1);
    const uint32_t b0l = movmatrix_t(l0), b1l = movmatrix_t(l1);
#pragma unroll
    for (int blk = 0; blk < KS; ++blk) {
      const uint4 v = *reinterpret_cast<const uint4*>(base + ((size_t)blk * 32 + lane) * 16);
      const uint32_t a[4] = {v.x, v.y, v.z, v.w};
      mma16816<BF16>(st.o[blk], a, b0h, b1h);
      mma16816<BF16>(st.o[blk], a, b0l, b1l);
    }
  } else {
    // bf16 tensor-core operands: centred codes (exact) and P scaled per token (hi + lo)
    LaneWords<TIER, D> lw;
    lw.load(base, lane);
    float s[2][NG], z[2][NG];
    load_meta<TIER, D>(base + codes_bytes(TIER, D), lane >> 2, s, z);
#pragma unroll
    for (int gi = 0; gi < NG; ++gi) {
      uint32_t h0, l0, h1, l1;
      split2<true>(p[0] * s[0][gi], p[1] * s[0][gi], h0, l0);
      split2<true>(p[2] * s[1][gi], p[3] * s[1][gi], h1, l1);
      const uint32_t b0h = movmatrix_t(h0), b1h = movmatrix_t(h1);
      const uint32_t b0l = movmatrix_t(l0), b1l = movmatrix_t(l1);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t a[4];
        lw.template frag<true>(2 * gi + h, a);
        mma16816<true>(st.o[2 * gi + h], a, b0h, b1h);
        mma16816<true>(st.o[2 * gi + h], a, b0l, b1l);
      }
      if constexpr (TIER != KVQ_TIER_I1 && TIER != KVQ_TIER_F8) {
        st.zacc[gi][0] += z[0][gi] * p[0] + z[1][gi] * p[2];
        st.zacc[gi][1] += z[0][gi] * p[1] + z[1][gi] * p[3];
      }
    }
  }
}

// ONLY16: the cache has 16-bit pages only (no code for the other tiers is generated, which
// keeps the kernel's instruction footprint small).
template <int D, bool BF16, bool ONLY16 = false>
__device__ __forceinline__ void process_page(const unsigned char* base, int tier, int nv, int lane, float scale_log2,
                                    WarpState<D>& st) {
  constexpr int KS = D / 16, NG = D / 32;
  float sacc[4] = {0.f, 0.f, 0.f, 0.f};
  if constexpr (ONLY16) {
    tier = KVQ_TIER_16;
    qk_page<KVQ_TIER_16, D, BF16>(base, lane, st, sacc);
  } else {
    switch (tier) {
      case KVQ_TIER_16: qk_page<KVQ_TIER_16, D, BF16>(base, lane, st, sacc); break;
      case KVQ_TIER_I8: qk_page<KVQ_TIER_I8, D, BF16>(base, lane, st, sacc); break;
      case KVQ_TIER_I4: qk_page<KVQ_TIER_I4, D, BF16>(base, lane, st, sacc); break;
      case KVQ_TIER_I2: qk_page<KVQ_TIER_I2, D, BF16>(base, lane, st, sacc); break;
      case KVQ_TIER_I1: qk_page<KVQ_TIER_I1, D, BF16>(base, lane, st, sacc); break;
      default: qk_page<KVQ_TIER_F8, D, BF16>(base, lane, st, sacc); break;
    }
  }
  const int t0 = lane >> 2, t1 = t0 + 8;
  float x[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) x[i] = sacc[i] * scale_log2;
  if (t0 >= nv) x[0] = x[1] = -INFINITY;
  if (t1 >= nv) x[2] = x[3] = -INFINITY;
  float pm0 = fmaxf(x[0], x[2]), pm1 = fmaxf(x[1], x[3]);
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    pm0 = fmaxf(pm0, __shfl_xor_sync(0xffffffffu, pm0, o));
    pm1 = fmaxf(pm1, __shfl_xor_sync(0xffffffffu, pm1, o));
  }
  const float mn0 = fmaxf(st.m[0], pm0), mn1 = fmaxf(st.m[1], pm1);
  const float a0 = ex2(st.m[0] - mn0), a1 = ex2(st.m[1] - mn1);
  float p[4];
  p[0] = ex2(x[0] - mn0);
  p[1] = ex2(x[1] - mn1);
  p[2] = ex2(x[2] - mn0);
  p[3] = ex2(x[3] - mn1);
  st.l[0] = st.l[0] * a0 + p[0] + p[2];
  st.l[1] = st.l[1] * a1 + p[1] + p[3];
  // rescale the accumulators only when some running maximum moved (else the factors are
  // exactly 1): after the first pages of a segment that is the rare case
  const bool moved = __any_sync(0xffffffffu, mn0 != st.m[0] || mn1 != st.m[1]);
  st.m[0] = mn0;
  st.m[1] = mn1;
  if (moved) {
#pragma unroll
    for (int blk = 0; blk < KS; ++blk) {
      st.o[blk][0] *= a0;
      st.o[blk][1] *= a1;
      st.o[blk][2] *= a0;
      st.o[blk][3] *= a1;
    }
#pragma unroll
    for (int gi = 0; gi < NG; ++gi) {
      st.zacc[gi][0] *= a0;
      st.zacc[gi][1] *= a1;
    }
  }
  const unsigned char* vbase = base + chunk_bytes(tier, D);
  if constexpr (ONLY16) {
    pv_page<KVQ_TIER_16, D, BF16>(vbase, lane, st, p);
    return;
  }
  switch (tier) {
    case KVQ_TIER_16: pv_page<KVQ_TIER_16, D, BF16>(vbase, lane, st, p); break;
    case KVQ_TIER_I8: pv_page<KVQ_TIER_I8, D, BF16>(vbase, lane, st, p); break;
    case KVQ_TIER_I4: pv_page<KVQ_TIER_I4, D, BF16>(vbase, lane, st, p); break;
    case KVQ_TIER_I2: pv_page<KVQ_TIER_I2, D, BF16>(vbase, lane, st, p); break;
    case KVQ_TIER_I1: pv_page<KVQ_TIER_I1, D, BF16>(vbase, lane, st, p); break;
    default: pv_page<KVQ_TIER_F8, D, BF16>(vbase, lane, st, p); break;
  }
}

// Load the segment's query fragments and per-group query sums; reset the state.
template <int D, bool BF16>
__device__ __forceinline__ void begin_segment(const uint16_t* q, int Hq, int G, int b, int g, int lane,
                                              WarpState<D>& st) {
  constexpr int KS = D / 16, NG = D / 32;
  const int g8 = lane >> 2, q4 = lane & 3;
  const uint16_t* qrow = q + ((size_t)b * Hq + (size_t)g * G + g8) * D;
  float part[NG];
#pragma unroll
  for (int gi = 0; gi < NG; ++gi) part[gi] = 0.f;
#pragma unroll
  for (int kk = 0; kk < KS; ++kk) {
    uint32_t b0 = 0, b1 = 0;
    if (g8 < G) {
      b0 = *reinterpret_cast<const uint32_t*>(qrow + 16 * kk + 2 * q4);
      b1 = *reinterpret_cast<const uint32_t*>(qrow + 16 * kk + 8 + 2 * q4);
    }
    st.qb[kk][0] = b0;
    st.qb[kk][1] = b1;
    part[kk / 2] += bits_to_float<BF16>(static_cast<uint16_t>(b0 & 0xFFFFu)) +
                    bits_to_float<BF16>(static_cast<uint16_t>(b0 >> 16)) +
                    bits_to_float<BF16>(static_cast<uint16_t>(b1 & 0xFFFFu)) +
                    bits_to_float<BF16>(static_cast<uint16_t>(b1 >> 16));
  }
#pragma unroll
  for (int gi = 0; gi < NG; ++gi) {
    float v = part[gi];
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    st.qs[gi][0] = __shfl_sync(0xffffffffu, v, 4 * (2 * q4));      // head 2*q4
    st.qs[gi][1] = __shfl_sync(0xffffffffu, v, 4 * (2 * q4 + 1));  // head 2*q4+1
    st.zacc[gi][0] = st.zacc[gi][1] = 0.f;
  }
  st.m[0] = st.m[1] = -INFINITY;
  st.l[0] = st.l[1] = 0.f;
#pragma unroll
  for (int blk = 0; blk < KS; ++blk) st.o[blk][0] = st.o[blk][1] = st.o[blk][2] = st.o[blk][3] = 0.f;
}

// Reduce the warp's (m, l, o) over its lanes and write it: o[h][d] at wo[h * D + d],
// (m, l) of head h at wml[2h], wml[2h + 1] (global or shared memory).
template <int D>
__device__ inline void write_warp_partial(int G, WarpState<D>& st, float* wo, float* wml, int lane) {
  constexpr int KS = D / 16;
  const int g8 = lane >> 2, q4 = lane & 3;
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    st.l[0] += __shfl_xor_sync(0xffffffffu, st.l[0], o);
    st.l[1] += __shfl_xor_sync(0xffffffffu, st.l[1], o);
#pragma unroll
    for (int gi = 0; gi < D / 32; ++gi) {
      st.zacc[gi][0] += __shfl_xor_sync(0xffffffffu, st.zacc[gi][0], o);
      st.zacc[gi][1] += __shfl_xor_sync(0xffffffffu, st.zacc[gi][1], o);
    }
  }
  const int h0 = 2 * q4, h1 = 2 * q4 + 1;
#pragma unroll
  for (int blk = 0; blk < KS; ++blk) {
    const int d0 = 16 * blk + g8, d1 = d0 + 8, gi = blk / 2;
    if (h0 < G) {
      wo[h0 * D + d0] = st.o[blk][0] + st.zacc[gi][0];
      wo[h0 * D + d1] = st.o[blk][2] + st.zacc[gi][0];
    }
    if (h1 < G) {
      wo[h1 * D + d0] = st.o[blk][1] + st.zacc[gi][1];
      wo[h1 * D + d1] = st.o[blk][3] + st.zacc[gi][1];
    }
  }
  if (g8 == 0) {
    if (h0 < G) { wml[h0 * 2] = st.m[0]; wml[h0 * 2 + 1] = st.l[0]; }
    if (h1 < G) { wml[h1 * 2] = st.m[1]; wml[h1 * 2 + 1] = st.l[1]; }
  }
}

}  // namespace kvq
