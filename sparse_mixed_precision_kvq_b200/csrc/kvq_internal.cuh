// Internal declarations shared by the libkvq translation units (device-side format,
// argument bundle, launch wrappers).  See include/kvq.h for the public contract.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

constexpr int kPage = 16;       // tokens per page
constexpr int kGroup = 32;      // channels per quantisation group
constexpr int kMaxG = 8;        // query heads per kv head handled by one mma N-tile
constexpr int kNumTiers = 5;
constexpr int kMaxSegments = 6144;  // B * Hkv limit of the attention kernel (offsets in shared memory)
// Head of every workspace: counters that must be zero when a call starts (every call
// leaves them zero); kvq_workspace_init zeroes it once.
constexpr size_t kCounterBytes = 65536;

__host__ __device__ inline int tier_bits(int tier) {
  return tier == 0 ? 16 : tier == 1 ? 8 : tier == 2 ? 4 : tier == 3 ? 2 : 1;
}
__host__ __device__ inline int codes_bytes(int tier, int D) { return kPage * D * tier_bits(tier) / 8; }
__host__ __device__ inline int meta_bytes(int tier, int D) {
  return tier == 0 ? 0 : kPage * (D / kGroup) * (tier == 4 ? 2 : 4);
}
__host__ __device__ inline int chunk_bytes(int tier, int D) { return codes_bytes(tier, D) + meta_bytes(tier, D); }

// Everything a kernel needs to locate pages (copied by value into kernel parameters).
struct DevCache {
  int B, Hq, Hkv, G, D, max_pages, dtype;
  const int32_t* block_table;
  const int32_t* seq_len;
  unsigned char* pool[kNumTiers];
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

__device__ inline void set_err(uint32_t* err, uint32_t bits) {
  if (err) atomicOr(err, bits);
}

// Decode a block-table entry; false (and an error bit) if tier or slot is invalid.
__device__ inline bool page_chunk(const DevCache& c, int b, int p, int g, int& tier,
                                  const unsigned char*& chunkK) {
  const uint32_t e = static_cast<uint32_t>(c.block_table[(size_t)b * c.max_pages + p]);
  tier = static_cast<int>(e >> 29);
  const long long slot = static_cast<long long>(e & 0x1FFFFFFFu);
  if (tier >= kNumTiers || c.pool[tier] == nullptr || slot >= c.pool_slots[tier]) {
    set_err(c.err, KVQ_DERR_BAD_PAGE);
    return false;
  }
  chunkK = c.pool[tier] + ((size_t)(slot * c.Hkv + g) * 2) * (size_t)c.chunk[tier];
  return true;
}

// 16-bit cache element <-> float/double
template <bool BF16>
__device__ inline float bits_to_float(uint16_t v) {
  if constexpr (BF16) return __uint_as_float(static_cast<uint32_t>(v) << 16);
  else return __half2float(__ushort_as_half(v));
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
int coverage_sort_size(const DevCache& c, const kvq_select_params& prm);
size_t attn_workspace_bytes(const DevCache& c, int num_ctas);
int attn_num_ctas(int device);
cudaError_t launch_attn(const DevCache& c, const void* q, const int32_t* sel, const int32_t* cnt, int kmax,
                        float sm_scale, void* out, float* lse, void* ws, int num_ctas, cudaStream_t s);
bool step_supported(const DevCache& c);
size_t step_workspace_bytes(const DevCache& c, int kmax);
cudaError_t launch_step(const DevCache& c, const int32_t* pos, const void* k_new, const void* v_new,
                        const void* q, const kvq_select_params& prm, float* scores, int32_t* sel, int32_t* cnt,
                        int kmax, float sm_scale, void* out, float* lse, void* ws, int num_ctas, cudaStream_t s);
cudaError_t launch_dequant(const DevCache& c, int b, int page, float* out, cudaStream_t s);
cudaError_t launch_requantize(const DevCache& c, const int32_t* items, int n, cudaStream_t s);

}  // namespace kvq
