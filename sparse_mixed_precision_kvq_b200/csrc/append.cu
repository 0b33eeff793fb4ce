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
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bg = blockIdx.x;
  const int b = bg / c.Hkv, g = bg % c.Hkv;
  griddep_wait();
  const int P = pos[b];
  if (P >= c.max_pages * kPage) {
    if (tid == 0) set_err(c.err, KVQ_DERR_BAD_POS);
  } else if (P >= 0) {
    const uint16_t* kr = k_new + (size_t)bg * c.D;
    const uint16_t* vr = v_new + (size_t)bg * c.D;
    const bool ok = append_phase1<BF16>(c, b, g, P, kr, tid, 128, nullptr);
    __syncthreads();
    if (ok) append_phase2<BF16>(c, b, g, P, kr, vr, warp, 4, lane);
  }
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

template <bool BF16>
__global__ void __launch_bounds__(128) requant_kernel(DevCache c, const int32_t* __restrict__ items) {
  const int g = blockIdx.y, tid = threadIdx.x;
  int b, p, n;
  uint32_t oe, ne;
  if (!requant_item(c, items, blockIdx.x, b, p, oe, ne, n)) {
    if (g == 0 && tid == 0) set_err(c.err, KVQ_DERR_BAD_PAGE);
    return;
  }
  const int D = c.D, ot = static_cast<int>(oe >> 29), nt = static_cast<int>(ne >> 29);
  const int OB = c.chunk[ot], NB = c.chunk[nt];
  const unsigned char* src = c.pool[ot] + ((size_t)(oe & 0x1FFFFFFFu) * c.Hkv + g) * 2 * (size_t)OB;
  unsigned char* dst = c.pool[nt] + ((size_t)(ne & 0x1FFFFFFFu) * c.Hkv + g) * 2 * (size_t)NB;

  __shared__ __align__(16) uint32_t old_words[2048];   // current K and V chunks (<= 8 KB)
  __shared__ __align__(16) uint32_t words[2][1024];    // new chunk images (<= 4 KB each)
  for (int k = tid; k < 2 * OB / 16; k += blockDim.x)
    reinterpret_cast<uint4*>(old_words)[k] = __ldcg(reinterpret_cast<const uint4*>(src) + k);
  for (int k = tid; k < 2 * 1024; k += blockDim.x) (&words[0][0])[k] = 0u;
  __syncthreads();

  const int warp = tid >> 5, lane = tid & 31, ng = D / kGroup;
  bool ov = false, nonfinite = false;
  for (int gi = warp; gi < 2 * n * ng; gi += 4) {
    const int kind = gi / (n * ng), rem = gi % (n * ng), t = rem / ng, grp = rem % ng;
    const int d = grp * kGroup + lane;
    const unsigned char* oc = reinterpret_cast<const unsigned char*>(old_words) + kind * OB;
    const double x = static_cast<double>(load_value(oc, kind, ot, D, BF16, t, d));
    nonfinite |= !isfinite(x);
    const QOut q = quant_group(x, nt, ov);
    int w, bit;
    elem_pos(kind, nt, D, t, d, w, bit);
    atomicOr(&words[kind][w], q.code << bit);
    if (lane == 0) {
      unsigned char* meta = reinterpret_cast<unsigned char*>(words[kind]) + codes_bytes(nt, D);
      if (nt == KVQ_TIER_I1)
        reinterpret_cast<uint16_t*>(meta)[t * ng + grp] = static_cast<uint16_t>(q.meta);
      else
        reinterpret_cast<uint32_t*>(meta)[t * ng + grp] = q.meta;
    }
  }
  __syncthreads();
  for (int kind = 0; kind < 2; ++kind) {
    const uint4* s4 = reinterpret_cast<const uint4*>(words[kind]);
    uint4* d4 = reinterpret_cast<uint4*>(dst + (size_t)kind * NB);
    for (int k = tid; k < NB / 16; k += blockDim.x) d4[k] = s4[k];
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
  if (c.dtype == KVQ_DT_BF16) requant_kernel<true><<<grid, 128, 0, s>>>(c, items);
  else requant_kernel<false><<<grid, 128, 0, s>>>(c, items);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  requant_commit_kernel<<<(n + 255) / 256, 256, 0, s>>>(c, items, n);
  return cudaGetLastError();
}

}  // namespace kvq
