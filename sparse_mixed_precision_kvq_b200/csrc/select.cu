// kvq_select_topk: per (sequence, kv head) page selection, one CTA each.
//
// AMASS "Quickstart" (budget: a fixed fraction of the pages is attended, here rounded
// up per sequence: k = ceil(P * bp / 10000)); ARGUS "Quickstart" (sink tokens kept) and
// "The One-Minute Explanation" (recent tokens stay hot): the first n_sink and last
// n_recent pages are always attended, in addition to the k best other pages.  Ranking:
// score descending, lower page index first among equal scores, NaN lowest.  The
// block-wide radix select lives in select_core.cuh (shared with the fused decode step).
#include <math.h>

#include "kvq_internal.cuh"
#include "select_core.cuh"

namespace kvq {
namespace {

struct SyncBar {
  __device__ bool operator()() const {
    __syncthreads();
    return true;
  }
};

// NT threads per (b, g): 512, or 1024 when a few long sequences leave most SMs idle.
// COV: coverage selection (its own instance, so that the top-k instance keeps its
// smaller register count).
template <int NT, bool COV>
__global__ void __launch_bounds__(NT) select_kernel(DevCache c, const float* __restrict__ scores,
                                                   kvq_select_params prm, int32_t* __restrict__ sel,
                                                   int32_t* __restrict__ cnt, int kmax, int ncov) {
  // keys [max_pages, rounded to 2 words]; coverage: then the candidates' mass keys [ncov] (u64)
  extern __shared__ __align__(16) uint32_t keys[];
  __shared__ SelShared sh;
  __shared__ __align__(16) uint32_t scratch[kSelScratchWords];
  const int bg = blockIdx.x;
  const int b = bg / c.Hkv;
  const int tid = threadIdx.x;
  // seq_len is an input of the call (no kernel of the step writes it): read through L2
  // before the wait, so that the score loads go out as soon as the scores are complete
  const int L = __ldcg(&c.seq_len[b]);
  griddep_wait();
  const int P = min((L + kPage - 1) / kPage, c.max_pages);
  const float* sc = scores + (size_t)bg * c.max_pages;
  constexpr bool topk = !COV;
  // while loading the keys, the range of the candidates' scores (the selection's first
  // pass) and the histogram's clearing, so that one barrier serves both
  bool nan_seen = false;
  // KB loads in flight per thread: rows of up to 8 * 512 (512 threads) or 9 * 1024 pages
  // (a 2^k-token context and its appended token) take one round trip
  constexpr int KB = NT >= 1024 ? 9 : 8;
  for (int p0 = tid; p0 < P; p0 += KB * NT) {
    float v[KB];
#pragma unroll
    for (int j = 0; j < KB; ++j) v[j] = p0 + j * NT < P ? sc[p0 + j * NT] : 0.f;
#pragma unroll
    for (int j = 0; j < KB; ++j)
      if (p0 + j * NT < P) keys[p0 + j * NT] = order_key(v[j], nan_seen);
  }
  if (nan_seen) set_err(c.err, KVQ_DERR_NAN_SCORE);
  constexpr bool kPre = NT <= 512;  // (the 1024-thread instance keeps the separate pass: registers)
  if (kPre && topk) {
    // this thread's own keys (no barrier needed to read them back)
    const SelectSplit sp = select_split(P, prm);
    float lo = INFINITY, hi = -INFINITY;
    for (int p = tid; p < sp.rs; p += NT) {
      if (p < sp.ns) continue;
      const uint32_t k = keys[p];
      if (k != 0u) {
        const float f = key_score(k);
        lo = fminf(lo, f);
        hi = fmaxf(hi, f);
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if ((tid & 31) == 0) {
      sh.wmin[tid >> 5] = lo;
      sh.wmax[tid >> 5] = hi;
    }
    for (int i = tid; i < 257; i += NT) scratch[i] = 0u;
    if (tid == 0) sh.ncand = 0;
  }
  __syncthreads();
  SyncBar bar;
  if constexpr (COV) {
    unsigned long long* mkey = reinterpret_cast<unsigned long long*>(keys + (c.max_pages + 1) / 2 * 2);
    select_coverage<NT>(keys, P, L, prm, mkey, scratch, sel + (size_t)bg * kmax, cnt + bg, kmax, c.err, sh, tid,
                        bar);
  } else {
    select_pages<NT, kPre>(keys, P, prm, sel + (size_t)bg * kmax, cnt + bg, kmax, c.err, scratch, sh, tid, bar);
  }
  griddep_launch_dependents();
}

template <int NT, bool COV>
cudaError_t launch_select_t(const DevCache& c, const float* scores, const kvq_select_params& prm, int32_t* sel,
                            int32_t* cnt, int kmax, int ncov, cudaStream_t s) {
  const size_t smem = (size_t)(c.max_pages + 1) / 2 * 2 * sizeof(uint32_t) + (size_t)ncov * 8;
  // static (histogram scratch) + dynamic (keys) shared memory may pass the 48 KB default
  cudaError_t e = cudaFuncSetAttribute(select_kernel<NT, COV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(select_kernel<NT, COV>, dim3(c.B * c.Hkv), dim3(NT), smem, s, c, scores, prm, sel, cnt, kmax,
                    ncov);
}

}  // namespace

// Mass-key slots coverage selection needs: the candidates of the longest possible
// sequence (max_pages minus the forced pages), at least 1; 0 if above kCovMaxCand or if
// the sequence's pages exceed kCovMaxPages.
int coverage_key_slots(const DevCache& c, const kvq_select_params& prm) {
  const int forced = max(prm.n_sink, 0) + max(prm.n_recent, 0);
  const int nc = max(1, c.max_pages - min(forced, c.max_pages));
  return nc <= kCovMaxCand && c.max_pages <= kCovMaxPages ? nc : 0;
}

cudaError_t launch_select(const DevCache& c, const float* scores, const kvq_select_params& prm,
                          int32_t* sel, int32_t* cnt, int kmax, cudaStream_t s) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  const bool wide = (long long)c.B * c.Hkv * 4 <= sm_count(dev) && c.max_pages >= 4096;
  const int ncov = prm.coverage_ppm > 0 ? coverage_key_slots(c, prm) : 0;
  if (ncov > 0)
    return wide ? launch_select_t<1024, true>(c, scores, prm, sel, cnt, kmax, ncov, s)
                : launch_select_t<512, true>(c, scores, prm, sel, cnt, kmax, ncov, s);
  return wide ? launch_select_t<1024, false>(c, scores, prm, sel, cnt, kmax, 0, s)
              : launch_select_t<512, false>(c, scores, prm, sel, cnt, kmax, 0, s);
}

}  // namespace kvq
