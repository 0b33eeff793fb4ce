// extern "C" entry points of libkvq (see include/kvq.h): host-side argument checks, then
// one or two kernel launches on the caller's stream.  No allocation, no synchronisation.
#include <stdint.h>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

// kvq_dequant_page: the value read back from storage for every element of one page.
__global__ void dequant_kernel(DevCache c, int b, int page, float* __restrict__ out) {
  const int g = blockIdx.x >> 1, kind = blockIdx.x & 1;
  const int D = c.D;
  int tier;
  const unsigned char *ck, *cv;
  if (!page_chunks(c, b, page, g, tier, ck, cv)) return;
  const unsigned char* chunk = kind ? cv : ck;
  for (int e = threadIdx.x; e < kPage * D; e += blockDim.x) {
    const int t = e / D, d = e % D;
    out[(((size_t)g * 2 + kind) * kPage + t) * D + d] = load_value(chunk, kind, tier, D, c.dtype == KVQ_DT_BF16, t, d);
  }
}

bool g_supported_g(int G) { return G == 1 || G == 2 || G == 4 || G == 8; }

kvq_status to_dev(const kvq_cache* k, DevCache& c) {
  if (k == nullptr) return KVQ_ERR_INVALID_ARG;
  if (k->B < 1 || k->Hq < 1 || k->Hkv < 1 || k->max_pages < 1 || k->Hq % k->Hkv != 0)
    return KVQ_ERR_INVALID_ARG;
  if (k->page_size != kPage || (k->D != 64 && k->D != 128)) return KVQ_ERR_UNSUPPORTED;
  if (k->dtype != KVQ_DT_F16 && k->dtype != KVQ_DT_BF16) return KVQ_ERR_UNSUPPORTED;
  if (!g_supported_g(k->Hq / k->Hkv)) return KVQ_ERR_UNSUPPORTED;
  if ((long long)k->B * k->Hkv > 65535) return KVQ_ERR_UNSUPPORTED;
  if (k->block_table == nullptr || k->seq_len == nullptr || k->summary == nullptr ||
      k->open_ksum == nullptr || k->err_word == nullptr)
    return KVQ_ERR_INVALID_ARG;
  c.B = k->B;
  c.Hq = k->Hq;
  c.Hkv = k->Hkv;
  c.G = k->Hq / k->Hkv;
  c.D = k->D;
  c.max_pages = k->max_pages;
  c.dtype = k->dtype;
  if (static_cast<uint32_t>(k->host_tiers) >> kNumTiers) return KVQ_ERR_INVALID_ARG;
  c.host_tiers = static_cast<uint32_t>(k->host_tiers);
  c.block_table = k->block_table;
  c.seq_len = k->seq_len;
  bool any = false;
  if (static_cast<uint32_t>(k->host_vtiers) >> kNumTiers || k->reserved0 != 0) return KVQ_ERR_INVALID_ARG;
  c.host_vtiers = static_cast<uint32_t>(k->host_vtiers);
  for (int t = 0; t < kNumTiers; ++t) {
    c.vpool[t] = static_cast<unsigned char*>(k->vpool[t]);
    if (k->vpool[t] && (k->pool[t] == nullptr || reinterpret_cast<uintptr_t>(k->vpool[t]) % 16 != 0))
      return KVQ_ERR_INVALID_ARG;
    if (((c.host_vtiers >> t) & 1u) && k->vpool[t] == nullptr) return KVQ_ERR_INVALID_ARG;
    c.pool[t] = static_cast<unsigned char*>(k->pool[t]);
    c.pool_slots[t] = k->pool[t] ? k->pool_slots[t] : 0;
    c.chunk[t] = chunk_bytes(t, k->D);
    if (k->pool[t] && (reinterpret_cast<uintptr_t>(k->pool[t]) % 16 != 0 || k->pool_slots[t] < 0))
      return KVQ_ERR_INVALID_ARG;
    any |= k->pool[t] != nullptr;
  }
  if (!any) return KVQ_ERR_INVALID_ARG;
  // the summary rows are read with 16-byte loads and bulk copies
  if (reinterpret_cast<uintptr_t>(k->summary) % 16 != 0) return KVQ_ERR_INVALID_ARG;
  c.summary = k->summary;
  c.open_ksum = k->open_ksum;
  c.err = k->err_word;
  return KVQ_OK;
}

kvq_status cuda_status(cudaError_t e) { return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA; }

bool aligned16(const void* p) { return reinterpret_cast<uintptr_t>(p) % 16 == 0; }

kvq_status to_quad(const kvq_quad* k, DevQuad& q) {
  if (k == nullptr || k->basis == nullptr || k->lambda == nullptr || k->open_sums == nullptr)
    return KVQ_ERR_INVALID_ARG;
  if (k->rank < 8 || k->rank > kMaxQuadRank || k->rank % 8 != 0) return KVQ_ERR_UNSUPPORTED;
  if (!aligned16(k->basis) || !aligned16(k->lambda) || reinterpret_cast<uintptr_t>(k->open_sums) % 8 != 0)
    return KVQ_ERR_INVALID_ARG;
  q.rank = k->rank;
  q.basis = k->basis;
  q.lambda = k->lambda;
  q.open = k->open_sums;
  return KVQ_OK;
}

int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) d = 0;
  return d;
}

}  // namespace
}  // namespace kvq

using namespace kvq;

extern "C" {

size_t kvq_chunk_bytes(int32_t tier, int32_t D) {
  if (tier < 0 || tier >= kNumTiers || (D != 64 && D != 128)) return 0;
  return static_cast<size_t>(chunk_bytes(tier, D));
}

const char* kvq_status_string(kvq_status s) {
  switch (s) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_INVALID_ARG: return "invalid argument";
    case KVQ_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case KVQ_ERR_WORKSPACE: return "workspace too small";
    case KVQ_ERR_CUDA: return "CUDA launch error";
  }
  return "unknown status";
}

kvq_status kvq_append(const kvq_cache* cache, const int32_t* pos, const void* k_new, const void* v_new,
                      kvq_stream_t stream) {
  DevCache c;
  kvq_status st = to_dev(cache, c);
  if (st != KVQ_OK) return st;
  if (pos == nullptr || k_new == nullptr || v_new == nullptr) return KVQ_ERR_INVALID_ARG;
  return cuda_status(launch_append(c, pos, k_new, v_new, reinterpret_cast<cudaStream_t>(stream)));
}

kvq_status kvq_build_pages(const kvq_cache* cache, const void* k_src, const void* v_src,
                           const int64_t* cu_seqlens, int64_t src_tokens, kvq_stream_t stream) {
  DevCache c;
  kvq_status st = to_dev(cache, c);
  if (st != KVQ_OK) return st;
  if (k_src == nullptr || v_src == nullptr || cu_seqlens == nullptr || src_tokens < 0) return KVQ_ERR_INVALID_ARG;
  return cuda_status(launch_build(c, k_src, v_src, cu_seqlens, src_tokens, reinterpret_cast<cudaStream_t>(stream)));
}

kvq_status kvq_page_scores(const kvq_cache* cache, const void* q, float* scores, kvq_stream_t stream) {
  DevCache c;
  kvq_status st = to_dev(cache, c);
  if (st != KVQ_OK) return st;
  if (q == nullptr || scores == nullptr || !aligned16(q)) return KVQ_ERR_INVALID_ARG;
  return cuda_status(launch_scores(c, q, scores, reinterpret_cast<cudaStream_t>(stream)));
}

kvq_status kvq_select_topk(const kvq_cache* cache, const float* scores, const kvq_select_params* params,
                           int32_t* sel, int32_t* cnt, int32_t kmax, kvq_stream_t stream) {
  DevCache c;
  kvq_status st = to_dev(cache, c);
  if (st != KVQ_OK) return st;
  if (scores == nullptr || params == nullptr || sel == nullptr || cnt == nullptr || kmax < 1)
    return KVQ_ERR_INVALID_ARG;
  if ((size_t)c.max_pages * 4 > 200 * 1024) return KVQ_ERR_UNSUPPORTED;  // keys in shared memory
  if (params->coverage_ppm > 0) {
    if (params->coverage_ppm > 1000000 || !(params->sm_scale > 0.f)) return KVQ_ERR_INVALID_ARG;
    const int n = coverage_key_slots(c, *params);
    if (n == 0 || ((size_t)c.max_pages + 1) / 2 * 8 + (size_t)n * 8 > 200 * 1024) return KVQ_ERR_UNSUPPORTED;
  }
  return cuda_status(launch_select(c, scores, *params, sel, cnt, kmax, reinterpret_cast<cudaStream_t>(stream)));
}

kvq_status kvq_workspace_size(const kvq_cache* cache, int32_t kmax, size_t* bytes) {
  DevCache c;
  kvq_status st = to_dev(cache, c);
  if (st != KVQ_OK) return st;
  if (bytes == nullptr || kmax < 1) return KVQ_ERR_INVALID_ARG;
  *bytes = attn_workspace_bytes(c, attn_grid(c, current_device()));
  return KVQ_OK;
}

kvq_status kvq_sparse_decode_attn(const kvq_cache* cache, const void* q, const int32_t* sel, const int32_t* cnt,
                                  int32_t kmax, float sm_scale, void* out, float* lse, void* workspace,
                                  size_t ws_bytes, kvq_stream_t stream) {
  DevCache c;
  kvq_status st = to_dev(cache, c);
  if (st != KVQ_OK) return st;
  if (q == nullptr || sel == nullptr || cnt == nullptr || out == nullptr || workspace == nullptr || kmax < 1)
    return KVQ_ERR_INVALID_ARG;
  if (!aligned16(workspace) || !(sm_scale > 0.f)) return KVQ_ERR_INVALID_ARG;
  if ((long long)c.B * c.Hkv >= kMaxSegments) return KVQ_ERR_UNSUPPORTED;  // offsets live in shared memory
  const int n = attn_grid(c, current_device());
  if (ws_bytes < attn_workspace_bytes(c, n)) return KVQ_ERR_WORKSPACE;
  return cuda_status(launch_attn(c, q, sel, cnt, kmax, sm_scale, out, lse, workspace, n,
                                 reinterpret_cast<cudaStream_t>(stream)));
}

kvq_status kvq_append_scores(const kvq_cache* cache, const int32_t* pos, const void* k_new, const void* v_new,
                             const void* q, float* scores, kvq_stream_t stream) {
  DevCache c;
  kvq_status st = to_dev(cache, c);
  if (st != KVQ_OK) return st;
  if (pos == nullptr || k_new == nullptr || v_new == nullptr || q == nullptr || scores == nullptr || !aligned16(q))
    return KVQ_ERR_INVALID_ARG;
  return cuda_status(launch_append_scores(c, pos, k_new, v_new, q, scores, reinterpret_cast<cudaStream_t>(stream)));
}

kvq_status kvq_score_select(const kvq_cache* cache, const int32_t* pos, const void* k_new, const void* v_new,
                            const void* q, const kvq_select_params* params, float* scores, int32_t* sel,
                            int32_t* cnt, int32_t kmax, void* workspace, size_t ws_bytes, kvq_stream_t stream) {
  DevCache c;
  kvq_status st = to_dev(cache, c);
  if (st != KVQ_OK) return st;
  if (q == nullptr || params == nullptr || scores == nullptr || sel == nullptr || cnt == nullptr ||
      workspace == nullptr || kmax < 1)
    return KVQ_ERR_INVALID_ARG;
  if (pos != nullptr && (k_new == nullptr || v_new == nullptr)) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(workspace)) return KVQ_ERR_INVALID_ARG;
  if (params->coverage_ppm > 0) return KVQ_ERR_UNSUPPORTED;
  if ((long long)c.B * c.Hkv > (long long)(kWaitLimitWord - kScoreSelectCounterWord)) return KVQ_ERR_UNSUPPORTED;
  if ((size_t)c.max_pages * 4 > 200 * 1024) return KVQ_ERR_UNSUPPORTED;  // keys in shared memory
  if (ws_bytes < kCounterBytes) return KVQ_ERR_WORKSPACE;
  unsigned* done = static_cast<unsigned*>(workspace) + kScoreSelectCounterWord;
  return cuda_status(launch_score_select(c, pos, k_new, v_new, q, *params, scores, sel, cnt, kmax, done,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

kvq_status kvq_step_workspace_size(const kvq_cache* cache, int32_t kmax, size_t* bytes) {
  DevCache c;
  kvq_status st = to_dev(cache, c);
  if (st != KVQ_OK) return st;
  if (bytes == nullptr || kmax < 1) return KVQ_ERR_INVALID_ARG;
  *bytes = step_workspace_bytes(c, kmax);
  return KVQ_OK;
}

kvq_status kvq_decode_step(const kvq_cache* cache, const int32_t* pos, const void* k_new, const void* v_new,
                           const void* q, const kvq_select_params* params, float* scores, int32_t* sel,
                           int32_t* cnt, int32_t kmax, float sm_scale, void* out, float* lse, void* workspace,
                           size_t ws_bytes, kvq_stream_t stream) {
  DevCache c;
  kvq_status st = to_dev(cache, c);
  if (st != KVQ_OK) return st;
  if (q == nullptr || params == nullptr || scores == nullptr || sel == nullptr || cnt == nullptr ||
      out == nullptr || workspace == nullptr || kmax < 1)
    return KVQ_ERR_INVALID_ARG;
  if (pos != nullptr && (k_new == nullptr || v_new == nullptr)) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(workspace) || !aligned16(q) || !(sm_scale > 0.f)) return KVQ_ERR_INVALID_ARG;
  if (params->coverage_ppm > 0) return KVQ_ERR_UNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(c.summary) % 16 != 0) return KVQ_ERR_INVALID_ARG;
  if (!step_supported(c)) return KVQ_ERR_UNSUPPORTED;
  if (ws_bytes < step_workspace_bytes(c, kmax)) return KVQ_ERR_WORKSPACE;
  return cuda_status(launch_step(c, pos, k_new, v_new, q, *params, scores, sel, cnt, kmax, sm_scale, out, lse,
                                 workspace, attn_num_ctas(current_device()), reinterpret_cast<cudaStream_t>(stream)));
}

kvq_status kvq_set_grid_override(int32_t ctas) {
  if (ctas < 0 || ctas > 65535) return KVQ_ERR_INVALID_ARG;
  set_grid_override(ctas);
  return KVQ_OK;
}

kvq_status kvq_workspace_init(void* workspace, size_t ws_bytes, kvq_stream_t stream) {
  if (workspace == nullptr || ws_bytes < kCounterBytes || !aligned16(workspace)) return KVQ_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(workspace, 0, kCounterBytes, reinterpret_cast<cudaStream_t>(stream)));
}

kvq_status kvq_quad_build(const kvq_cache* cache, const kvq_quad* quad, const void* k_src,
                          const int64_t* cu_seqlens, int64_t src_tokens, kvq_stream_t stream) {
  DevCache c;
  DevQuad q;
  kvq_status st = to_dev(cache, c);
  if (st == KVQ_OK) st = to_quad(quad, q);
  if (st != KVQ_OK) return st;
  if (k_src == nullptr || cu_seqlens == nullptr || src_tokens < 0) return KVQ_ERR_INVALID_ARG;
  return cuda_status(launch_quad_build(c, q, k_src, cu_seqlens, src_tokens, reinterpret_cast<cudaStream_t>(stream)));
}

kvq_status kvq_quad_append(const kvq_cache* cache, const kvq_quad* quad, const int32_t* pos, const void* k_new,
                           kvq_stream_t stream) {
  DevCache c;
  DevQuad q;
  kvq_status st = to_dev(cache, c);
  if (st == KVQ_OK) st = to_quad(quad, q);
  if (st != KVQ_OK) return st;
  if (pos == nullptr || k_new == nullptr) return KVQ_ERR_INVALID_ARG;
  return cuda_status(launch_quad_append(c, q, pos, k_new, reinterpret_cast<cudaStream_t>(stream)));
}

kvq_status kvq_quad_page_scores(const kvq_cache* cache, const kvq_quad* quad, const void* q, float sm_scale,
                                float* scores, kvq_stream_t stream) {
  DevCache c;
  DevQuad qd;
  kvq_status st = to_dev(cache, c);
  if (st == KVQ_OK) st = to_quad(quad, qd);
  if (st != KVQ_OK) return st;
  if (q == nullptr || scores == nullptr || !aligned16(q) || !(sm_scale > 0.0f)) return KVQ_ERR_INVALID_ARG;
  return cuda_status(
      launch_quad_scores(c, qd, q, sm_scale, scores, nullptr, nullptr, nullptr, reinterpret_cast<cudaStream_t>(stream)));
}

kvq_status kvq_quad_append_scores(const kvq_cache* cache, const kvq_quad* quad, const int32_t* pos,
                                  const void* k_new, const void* v_new, const void* q, float sm_scale, float* scores,
                                  kvq_stream_t stream) {
  DevCache c;
  DevQuad qd;
  kvq_status st = to_dev(cache, c);
  if (st == KVQ_OK) st = to_quad(quad, qd);
  if (st != KVQ_OK) return st;
  if (pos == nullptr || k_new == nullptr || v_new == nullptr) return KVQ_ERR_INVALID_ARG;
  if (q == nullptr || scores == nullptr || !aligned16(q) || !(sm_scale > 0.0f)) return KVQ_ERR_INVALID_ARG;
  return cuda_status(launch_quad_scores(c, qd, q, sm_scale, scores, pos, k_new, v_new,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

kvq_status kvq_requantize_pages(const kvq_cache* cache, const int32_t* items, int32_t n, kvq_stream_t stream) {
  DevCache c;
  kvq_status st = to_dev(cache, c);
  if (st != KVQ_OK) return st;
  if (n < 0 || (n > 0 && items == nullptr)) return KVQ_ERR_INVALID_ARG;
  if (n == 0) return KVQ_OK;
  return cuda_status(launch_requantize(c, items, n, reinterpret_cast<cudaStream_t>(stream)));
}

kvq_status kvq_dequant_page(const kvq_cache* cache, int32_t b, int32_t page, float* out, kvq_stream_t stream) {
  DevCache c;
  kvq_status st = to_dev(cache, c);
  if (st != KVQ_OK) return st;
  if (out == nullptr || b < 0 || b >= c.B || page < 0 || page >= c.max_pages) return KVQ_ERR_INVALID_ARG;
  dequant_kernel<<<c.Hkv * 2, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(c, b, page, out);
  return cuda_status(cudaGetLastError());
}

}  // extern "C"
