// Internal declarations shared by the libkvq translation units (device-side format,
// argument bundle, launch wrappers).  See include/kvq.h for the public contract.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

constexpr int kPage = 16;       // tokens per page
constexpr int kGroup = 32;      // channels per quantisation group
constexpr int kMaxG = 8;        // query heads per kv head handled by one mma N-tile
constexpr int kNumTiers = 6;
// B * Hkv limit of the attention kernel: its segment offsets and completion list live in
// shared memory beside the one-CTA-per-SM 24 KB-per-warp page rings (196,608 + 1,792 +
// 6 * B*Hkv bytes, within the 227 KB a CTA may hold up to 5,651 segments)
constexpr int kMaxSegments = 5632;
// Head of every workspace: counters that must be zero when a call starts (every call
// leaves them zero); kvq_workspace_init zeroes it once.
constexpr size_t kCounterBytes = 65536;
// Last word of that head: the limit of every bounded wait of a call on this workspace, in
// microseconds (0: the default, kWaitNs).  No counter ever uses it.
constexpr int kWaitLimitWord = static_cast<int>(kCounterBytes / 4) - 1;

__host__ __device__ constexpr int tier_bits(int tier) {
  return tier == 0 ? 16 : tier == 1 ? 8 : tier == 2 ? 4 : tier == 3 ? 2 : tier == 4 ? 1 : 8;
}
__host__ __device__ constexpr int codes_bytes(int tier, int D) { return kPage * D * tier_bits(tier) / 8; }
__host__ __device__ constexpr int meta_bytes(int tier, int D) {
  return tier == 0 ? 0 : kPage * (D / kGroup) * ((tier == 4 || tier == 5) ? 2 : 4);
}
__host__ __device__ constexpr int chunk_bytes(int tier, int D) { return codes_bytes(tier, D) + meta_bytes(tier, D); }

// quad page-score state (see kvq_quad in kvq.h).
constexpr int kMaxQuadRank = 32;
struct DevQuad {
  int rank;
  const float* basis;
  uint16_t* lambda;
  double* open;
};

// Everything a kernel needs to locate pages (copied by value into kernel parameters).
struct DevCache {
  int B, Hq, Hkv, G, D, max_pages, dtype;
  uint32_t host_tiers;  // bit t: pool t is pinned host memory mapped into the device address space
  const int32_t* block_table;
  const int32_t* seq_len;
  unsigned char* pool[kNumTiers];
  unsigned char* vpool[kNumTiers];  // separate V chunks of a tier (nullptr: V next to K in pool)
  uint32_t host_vtiers;             // bit t: vpool t is pinned host memory
  long long pool_slots[kNumTiers];
  int chunk[kNumTiers];  // chunk bytes per tier
  uint16_t* summary;
  double* open_ksum;
  uint32_t* err;
};

// Position of element (t, d) of a K (kind 0) or V (kind 1) chunk: the uint32 word of the
// codes area and the bit offset of its code (16-bit tier: offset 0 or 16 of the value).
__host__ __device__ inline void elem_pos(int kind, int tier, int D, int t, int d, int& word, int& bit) {
  const int kk = d >> 4, c = d & 15;
  int lam, r, h;
  if (kind == 0) {
    lam = 4 * (t & 7) + ((c & 7) >> 1);
    r = 2 * (c >> 3) + (t >> 3);
    h = c & 1;
  } else {
    lam = 4 * (c & 7) + ((t & 7) >> 1);
    r = 2 * (t >> 3) + (c >> 3);
    h = t & 1;
  }
  if (tier == 0) {
    word = (kk * 32 + lam) * 4 + r;
    bit = 16 * h;
    return;
  }
  const int b = tier_bits(tier);
  const int ppw = 16 / b;
  const int R = 4 * kk + r;
  const int w = R / ppw, j = R % ppw;
  const int nw = D * b / 64;
  const int pw = nw < 4 ? nw : 4;
  word = ((w / pw) * 32 + lam) * pw + (w % pw);
  bit = b * j + 16 * h;
}

// Token t and channel c (0..15 within the 16-channel block) of fragment lane `lam`,
// register `r`, half `h` of a K (KIND 0) or V (KIND 1) chunk: the inverse of elem_pos.
template <int KIND>
__host__ __device__ constexpr void frag_tc(int lam, int r, int h, int& t, int& c) {
  if (KIND == 0) {
    t = 8 * (r & 1) + (lam >> 2);
    c = 8 * (r >> 1) + 2 * (lam & 3) + h;
  } else {
    c = 8 * (r & 1) + (lam >> 2);
    t = 8 * (r >> 1) + 2 * (lam & 3) + h;
  }
}

// Every element stored in word W of a chunk's codes area: f(t, d, shift) for each, shift
// being the bit offset of its code (16-bit tier: of its value) in the word.
template <int TIER, int KIND, int D, typename F>
__host__ __device__ inline void word_elems(int W, F&& f) {
  if constexpr (TIER == 0) {
    const int kk = W >> 7, lam = (W >> 2) & 31, r = W & 3;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      int t = 0, c = 0;
      frag_tc<KIND>(lam, r, h, t, c);
      f(t, 16 * kk + c, 16 * h);
    }
  } else {
    constexpr int b = tier_bits(TIER), ppw = 16 / b, nw = D * b / 64, pw = nw < 4 ? nw : 4;
    const int lam = (W / pw) & 31, w = (W / (32 * pw)) * pw + W % pw;
#pragma unroll
    for (int j = 0; j < ppw; ++j) {
      const int R = w * ppw + j, kk = R >> 2, r = R & 3;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        int t = 0, c = 0;
        frag_tc<KIND>(lam, r, h, t, c);
        f(t, 16 * kk + c, b * j + 16 * h);
      }
    }
  }
}

// word_elems for word W = W0 + 128 * i of a chunk's codes area (0 <= W0 < 128, i a
// compile-time constant after unrolling): the position inside the word's 128-word block
// fixes lam, r and the pair index modulo 4, so only a constant offset depends on i.
template <int TIER, int KIND, int D, int I, typename F>
__host__ __device__ inline void word_elems_at(int W0, F&& f) {
  if constexpr (TIER == 0) {
    const int lam = (W0 >> 2) & 31, r = W0 & 3;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      int t = 0, c = 0;
      frag_tc<KIND>(lam, r, h, t, c);
      f(t, 16 * I + c, 16 * h);
    }
  } else {
    constexpr int b = tier_bits(TIER), ppw = 16 / b, nw = D * b / 64, pw = nw < 4 ? nw : 4;
    const int lam = (W0 / pw) & 31, w = (W0 / (32 * pw)) * pw + W0 % pw + 4 * I;
#pragma unroll
    for (int j = 0; j < ppw; ++j) {
      const int R = w * ppw + j, kk = R >> 2, r = R & 3;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        int t = 0, c = 0;
        frag_tc<KIND>(lam, r, h, t, c);
        f(t, 16 * kk + c, b * j + 16 * h);
      }
    }
  }
}

__device__ inline void set_err(uint32_t* err, uint32_t bits) {
  if (err) atomicOr(err, bits);
}

// K and V chunks of (slot, kv head g) in tier `tier`: adjacent in pool[tier], or, with a
// separate V pool, at the same offset in pool[tier] and vpool[tier].
__device__ inline void slot_chunks(const DevCache& c, int tier, long long slot, int g, const unsigned char*& chunkK,
                                   const unsigned char*& chunkV) {
  const size_t i = (size_t)slot * c.Hkv + g, cb = (size_t)c.chunk[tier];
  if (c.vpool[tier] != nullptr) {
    chunkK = c.pool[tier] + i * cb;
    chunkV = c.vpool[tier] + i * cb;
  } else {
    chunkK = c.pool[tier] + 2 * i * cb;
    chunkV = chunkK + cb;
  }
}

// Decode a block-table entry into the page's K and V chunks; false (and an error bit) if
// tier or slot is invalid.
__device__ inline bool page_chunks(const DevCache& c, int b, int p, int g, int& tier, const unsigned char*& chunkK,
                                   const unsigned char*& chunkV) {
  const uint32_t e = static_cast<uint32_t>(c.block_table[(size_t)b * c.max_pages + p]);
  tier = static_cast<int>(e >> 29);
  const long long slot = static_cast<long long>(e & 0x1FFFFFFFu);
  if (tier >= kNumTiers || c.pool[tier] == nullptr || slot >= c.pool_slots[tier]) {
    set_err(c.err, KVQ_DERR_BAD_PAGE);
    return false;
  }
  slot_chunks(c, tier, slot, g, chunkK, chunkV);
  return true;
}

// 16-bit cache element <-> float/double
template <bool BF16>
__device__ inline float bits_to_float(uint16_t v) {
  if constexpr (BF16) return __uint_as_float(static_cast<uint32_t>(v) << 16);
  else return __half2float(__ushort_as_half(v));
}

// FP8 e4m3 code -> float (exact, NaN codes -> NaN).
__device__ inline float e4m3_to_float(uint32_t code) {
  return __half2float(__half(__nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(code), __NV_E4M3)));
}

// Value read back from storage for element (t, d) of a K (kind 0) or V (kind 1) chunk:
// the 16-bit value, fp32(c * scale + zero) with one rounding, or +-m.
__device__ inline float load_value(const unsigned char* chunk, int kind, int tier, int D, bool bf16, int t, int d) {
  int w, bit;
  elem_pos(kind, tier, D, t, d, w, bit);
  const uint32_t word = reinterpret_cast<const uint32_t*>(chunk)[w];
  if (tier == 0) {
    const uint16_t x = static_cast<uint16_t>(word >> bit);
    return bf16 ? bits_to_float<true>(x) : bits_to_float<false>(x);
  }
  const int ng = D / kGroup;
  const uint32_t code = (word >> bit) & ((1u << tier_bits(tier)) - 1u);
  const unsigned char* meta = chunk + codes_bytes(tier, D);
  if (tier == 4) {
    const float m = __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(meta)[t * ng + d / kGroup]));
    return code ? m : -m;
  }
  if (tier == 5) {  // e4m3 value times the group's fp16 scale (exact in fp32)
    const float sc = __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(meta)[t * ng + d / kGroup]));
    return e4m3_to_float(code) * sc;
  }
  const uint32_t mw = reinterpret_cast<const uint32_t*>(meta)[t * ng + d / kGroup];
  const float scale = __half2float(__ushort_as_half(static_cast<uint16_t>(mw & 0xFFFFu)));
  const float zero = __half2float(__ushort_as_half(static_cast<uint16_t>(mw >> 16)));
  return fmaf(static_cast<float>(code), scale, zero);
}

// fp16 round-half-even of a double, saturating at +-65504 (flag in *ov).
__device__ inline uint16_t fp16_sat(double v, bool& ov) {
  __half h = __double2half(v);
  uint16_t bits = __half_as_ushort(h);
  if ((bits & 0x7FFFu) == 0x7C00u && !isinf(v)) {  // finite value rounded to +-inf
    ov = true;
    bits = (bits & 0x8000u) | 0x7BFFu;
  }
  return bits;
}

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start while the previous kernel in the stream finishes; it must call
// griddep_wait() before touching anything that kernel wrote, and calls
// griddep_launch_dependents() once its own dependents may start launching.
__device__ inline void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ inline void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Launch wrappers (defined in the .cu files).
cudaError_t launch_append(const DevCache& c, const int32_t* pos, const void* k_new, const void* v_new,
                          cudaStream_t s);
cudaError_t launch_build(const DevCache& c, const void* k_src, const void* v_src, const int64_t* cu,
                         int64_t src_tokens, cudaStream_t s);
cudaError_t launch_scores(const DevCache& c, const void* q, float* scores, cudaStream_t s);
cudaError_t launch_score_select(const DevCache& c, const int32_t* pos, const void* k_new, const void* v_new,
                                const void* q, const kvq_select_params& prm, float* scores, int32_t* sel,
                                int32_t* cnt, int kmax, unsigned* done, cudaStream_t s);
cudaError_t launch_append_scores(const DevCache& c, const int32_t* pos, const void* k_new, const void* v_new,
                                 const void* q, float* scores, cudaStream_t s);
constexpr size_t kScoreSelectCounterWord = 8192;  // workspace word of the per-(b, g) tile counters
cudaError_t launch_select(const DevCache& c, const float* scores, const kvq_select_params& prm,
                          int32_t* sel, int32_t* cnt, int kmax, cudaStream_t s);
int coverage_key_slots(const DevCache& c, const kvq_select_params& prm);
size_t attn_workspace_bytes(const DevCache& c, int num_ctas);
int sm_count(int device);      // streaming multiprocessors of the device (cached)
int attn_num_ctas(int device);  // grid of the fused step: sm_count, or the override
int attn_grid(const DevCache& c, int device);  // grid of the attention kernel for this cache (or the override)
void set_grid_override(int ctas);
cudaError_t launch_attn(const DevCache& c, const void* q, const int32_t* sel, const int32_t* cnt, int kmax,
                        float sm_scale, void* out, float* lse, void* ws, int num_ctas, cudaStream_t s);
bool step_supported(const DevCache& c);
size_t step_workspace_bytes(const DevCache& c, int kmax);
cudaError_t launch_step(const DevCache& c, const int32_t* pos, const void* k_new, const void* v_new,
                        const void* q, const kvq_select_params& prm, float* scores, int32_t* sel, int32_t* cnt,
                        int kmax, float sm_scale, void* out, float* lse, void* ws, int num_ctas, cudaStream_t s);
cudaError_t launch_dequant(const DevCache& c, int b, int page, float* out, cudaStream_t s);
cudaError_t launch_requantize(const DevCache& c, const int32_t* items, int n, cudaStream_t s);
cudaError_t launch_quad_build(const DevCache& c, const DevQuad& qd, const void* k_src, const int64_t* cu,
                              int64_t src_tokens, cudaStream_t s);
cudaError_t launch_quad_append(const DevCache& c, const DevQuad& qd, const int32_t* pos, const void* k_new,
                               cudaStream_t s);
cudaError_t launch_quad_scores(const DevCache& c, const DevQuad& qd, const void* q, float sm_scale, float* scores,
                               const int32_t* pos, const void* k_new, const void* v_new, cudaStream_t s);

}  // namespace kvq
