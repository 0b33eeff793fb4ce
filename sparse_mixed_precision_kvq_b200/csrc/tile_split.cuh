// Division of the page-score sweeps' 16-page tiles among warps.
//
// A (sequence, kv head) row of P pages has ceil(P / 16) tiles that hold pages; a ragged
// batch leaves most of a max_pages row empty, so the sweeps divide only those tiles among
// the warps.  Each CTA builds the tile counts' exclusive prefix over the B * Hkv rows in
// shared memory (from seq_len, an input of the call, read through L2 so that it may run
// before the grid waits on the previous kernel); item i of the flat list is tile
// i - pre[bg] of the last row bg with pre[bg] <= i.  The scores past a row's tiles are
// -inf, written by a separate fill.
#pragma once

#include "kvq_internal.cuh"

namespace kvq {

// Pages [0, P) of row bg that the sweeps score.
__device__ inline int row_pages(const DevCache& c, int bg) {
  const int L = __ldcg(&c.seq_len[bg / c.Hkv]);
  return min(max((L + kPage - 1) / kPage, 0), c.max_pages);
}

// pre[0 .. B * Hkv] (shared memory): the exclusive prefix of the rows' tile counts, the
// total in pre[B * Hkv].  All NT threads of the CTA call it; s_part holds NT / 32 ints.
// Ends with a barrier.
template <int NT>
__device__ inline int row_tile_prefix(const DevCache& c, int* pre, int* s_part, int tid) {
  constexpr int NW = NT / 32;
  const int BH = c.B * c.Hkv, lane = tid & 31, warp = tid >> 5;
  const int per = (BH + NT - 1) / NT;
  const int lo = min(BH, tid * per), hi = min(BH, lo + per);
  int s = 0;
  for (int bg = lo; bg < hi; ++bg) {
    const int t = (row_pages(c, bg) + 15) / 16;
    pre[bg] = t;
    s += t;
  }
  int x = s;  // inclusive prefix over the warp's lanes
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_part[warp] = x;
  __syncthreads();
  int run = x - s, all = 0;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const int v = s_part[w];
    if (w < warp) run += v;
    all += v;
  }
  for (int bg = lo; bg < hi; ++bg) {
    const int t = pre[bg];
    pre[bg] = run;
    run += t;
  }
  if (tid == 0) pre[BH] = all;
  __syncthreads();
  return all;
}

// The row of flat item i (0 <= i < pre[BH]): the last bg with pre[bg] <= i.
__device__ inline int row_of_item(const int* pre, int BH, int i) {
  int lo = 0, hi = BH - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pre[mid] <= i) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// The same with a forward cursor over increasing items: advances cur to item i's row.
__device__ inline int advance_row(const int* pre, int& cur, int i) {
  while (pre[cur + 1] <= i) ++cur;
  return cur;
}

// -inf for every page of row bg from its first page past the scored tiles to max_pages,
// rows gw, gw + nw, ... (one warp each).
__device__ inline void fill_past_tiles(const DevCache& c, const int* pre, float* scores, int gw, int nw, int lane) {
  const int BH = c.B * c.Hkv;
  for (int bg = gw; bg < BH; bg += nw) {
    float* row = scores + (size_t)bg * c.max_pages;
    for (int p = (pre[bg + 1] - pre[bg]) * 16 + lane; p < c.max_pages; p += 32) row[p] = -INFINITY;
  }
}

}  // namespace kvq
