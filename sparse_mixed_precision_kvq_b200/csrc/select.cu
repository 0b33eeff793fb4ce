// kvq_select_topk: per (sequence, kv head) page selection.
//
// AMASS "Quickstart" (budget: a fixed fraction of the pages is attended, here rounded
// up per sequence: k = ceil(P * bp / 10000)); ARGUS "Quickstart" (sink tokens kept) and
// "The One-Minute Explanation" (recent tokens stay hot): the first n_sink and last
// n_recent pages are always attended, in addition to the k best other pages.  Ranking:
// score descending, lower page index first among equal scores, NaN lowest.
//
// One CTA per (b, g).  Scores are mapped to order-preserving 32-bit keys in shared
// memory; an exact MSB-first radix select (4 passes of 8 bits, shared-memory histograms)
// finds the k-th largest key; pages with a larger key, the lowest-indexed pages with an
// equal key, and the forced pages are then emitted in ascending order with two block
// scans.  No floating-point decision is re-taken: ties are resolved on the keys.
#include <math.h>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kSelThreads = 512;

__device__ inline uint32_t order_key(float f, bool& nan) {
  if (isnan(f)) {
    nan = true;
    return 0u;
  }
  if (f == 0.0f) f = 0.0f;  // -0 and +0 rank equal
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive block-wide prefix sum of one int per thread; *total receives the sum.
__device__ inline int block_exclusive_scan(int v, int* sh, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kSelThreads / 32 ? sh[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kSelThreads / 32) sh[lane] = w;
  }
  __syncthreads();
  const int before = (warp ? sh[warp - 1] : 0) + x - v;
  *total = sh[kSelThreads / 32 - 1];
  __syncthreads();
  return before;
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(DevCache c, const float* __restrict__ scores,
                                                             kvq_select_params prm, int32_t* __restrict__ sel,
                                                             int32_t* __restrict__ cnt, int kmax) {
  extern __shared__ uint32_t keys[];  // [max_pages]
  __shared__ int hist[256];
  __shared__ int scan_sh[kSelThreads / 32];
  __shared__ uint32_t s_prefix;
  __shared__ int s_rem;

  const int bg = blockIdx.x;
  const int b = bg / c.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  griddep_wait();
  const int L = c.seq_len[b];
  const int P = min((L + kPage - 1) / kPage, c.max_pages);
  const float* sc = scores + (size_t)bg * c.max_pages;

  const int ns = min(max(prm.n_sink, 0), P);
  const int rs = max(P - max(prm.n_recent, 0), 0);
  const int nF = ns + (P - rs) - max(0, ns - rs);
  const int nC = P - nF;
  const long long kb = prm.k_abs >= 0 ? (long long)prm.k_abs
                                      : ((long long)P * prm.k_frac_bp + 9999) / 10000;
  const long long kb0 = kb < 0 ? 0 : kb;
  const int kk = static_cast<int>(kb0 < nC ? kb0 : nC);

  bool nan_seen = false;
  for (int p = tid; p < P; p += kSelThreads) keys[p] = order_key(sc[p], nan_seen);
  if (nan_seen) set_err(c.err, KVQ_DERR_NAN_SCORE);
  __syncthreads();

  // mode 0: no candidate chosen, 1: every candidate, 2: by threshold key
  const int mode = (kk == 0) ? 0 : (kk == nC ? 1 : 2);
  uint32_t thr = 0;
  int need = 0;
  if (mode == 2) {
    uint32_t prefix = 0;
    int rem = kk;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
      __syncthreads();
      const uint32_t hmask = (shift == 24) ? 0u : (0xFFFFFFFFu << (shift + 8));
      // warp-aggregated: one shared atomic per distinct bin per warp instruction (most keys
      // share their top bytes, so plain atomics would serialise on one or two bins)
      for (int base = warp * 32; base < P; base += kSelThreads) {
        const int p = base + lane;
        bool active = false;
        uint32_t bin = 256u;
        if (p < P && !(p < ns || p >= rs)) {
          const uint32_t k = keys[p];
          if ((k & hmask) == (prefix & hmask)) {
            active = true;
            bin = (k >> shift) & 255u;
          }
        }
        const unsigned peers = __match_any_sync(0xffffffffu, bin);
        if (active && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
      }
      __syncthreads();
      if (warp == 0) {
        int h8[8], tot = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          h8[i] = hist[lane * 8 + i];
          tot += h8[i];
        }
        int suf = tot;  // sum over lanes >= lane
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_down_sync(0xffffffffu, suf, o);
          if (lane + o < 32) suf += y;
        }
        int cum = suf - tot;  // keys in bins above this lane's bins
#pragma unroll
        for (int i = 7; i >= 0; --i) {
          const int nxt = cum + h8[i];
          if (cum < rem && rem <= nxt) {
            s_prefix = prefix | (static_cast<uint32_t>(lane * 8 + i) << shift);
            s_rem = rem - cum;
          }
          cum = nxt;
        }
      }
      __syncthreads();
      prefix = s_prefix;
      rem = s_rem;
      __syncthreads();
    }
    thr = prefix;
    need = rem;
  }

  // contiguous page chunk per thread, emitted in ascending order
  const int CH = (P + kSelThreads - 1) / kSelThreads;
  const int lo = min(P, tid * CH), hi = min(P, lo + CH);
  int eq = 0;
  if (mode == 2)
    for (int p = lo; p < hi; ++p)
      if (!(p < ns || p >= rs) && keys[p] == thr) ++eq;
  int tot_eq;
  const int eq_before = block_exclusive_scan(eq, scan_sh, &tot_eq);

  auto chosen = [&](int p, int& e) -> bool {
    if (p < ns || p >= rs) return true;
    if (mode == 1) return true;
    if (mode == 0) return false;
    const uint32_t k = keys[p];
    if (k > thr) return true;
    if (k == thr) return (e++) < need;
    return false;
  };
  int nsel = 0, e = eq_before;
  for (int p = lo; p < hi; ++p) nsel += chosen(p, e) ? 1 : 0;
  int total;
  int off = block_exclusive_scan(nsel, scan_sh, &total);
  e = eq_before;
  int32_t* out = sel + (size_t)bg * kmax;
  for (int p = lo; p < hi; ++p) {
    if (chosen(p, e)) {
      if (off < kmax) out[off] = p;
      ++off;
    }
  }
  if (tid == 0) {
    cnt[bg] = min(total, kmax);
    if (total > kmax) set_err(c.err, KVQ_DERR_KMAX);
  }
  griddep_launch_dependents();
}

}  // namespace

cudaError_t launch_select(const DevCache& c, const float* scores, const kvq_select_params& prm,
                          int32_t* sel, int32_t* cnt, int kmax, cudaStream_t s) {
  const size_t smem = (size_t)c.max_pages * sizeof(uint32_t);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(select_kernel, dim3(c.B * c.Hkv), dim3(kSelThreads), smem, s, c, scores, prm, sel, cnt, kmax);
}

}  // namespace kvq
