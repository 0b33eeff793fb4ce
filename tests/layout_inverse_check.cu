// Host program: word_elems (the decoder of a packed chunk word, used by the re-quantiser)
// is the exact inverse of elem_pos (the writer's element -> word/bit map) for every tier,
// K and V, D = 64 and 128: each element of a chunk is produced by exactly one word slot,
// and elem_pos sends it back to that word and bit; word_elems_at (the same decoder with
// the word split as W0 + 128 * i) lists the same elements.  Exit status 0 when they agree.
#include <cstdio>
#include <utility>

#include "kvq_internal.cuh"

using namespace kvq;

template <int TIER, int KIND, int D>
int mismatches() {
  static int seen[kPage][128];
  for (auto& row : seen)
    for (auto& x : row) x = 0;
  int bad = 0;
  for (int W = 0; W < codes_bytes(TIER, D) / 4; ++W)
    word_elems<TIER, KIND, D>(W, [&](int t, int d, int sh) {
      int w = -1, bit = -1;
      elem_pos(KIND, TIER, D, t, d, w, bit);
      if (t < 0 || t >= kPage || d < 0 || d >= D || w != W || bit != sh) ++bad;
      else ++seen[t][d];
    });
  for (int t = 0; t < kPage; ++t)
    for (int d = 0; d < D; ++d) bad += seen[t][d] != 1;
  return bad;
}

// word_elems_at<..., I>(W0) must list the same elements as word_elems(W0 + 128 * I).
template <int TIER, int KIND, int D, int I>
int split_mismatches() {
  int bad = 0;
  for (int W0 = 0; W0 < 128 && W0 + 128 * I < codes_bytes(TIER, D) / 4; ++W0) {
    int a[64][3], na = 0, nb = 0;
    word_elems<TIER, KIND, D>(W0 + 128 * I, [&](int t, int d, int sh) {
      a[na][0] = t, a[na][1] = d, a[na][2] = sh;
      ++na;
    });
    word_elems_at<TIER, KIND, D, I>(W0, [&](int t, int d, int sh) {
      bad += nb >= na || a[nb][0] != t || a[nb][1] != d || a[nb][2] != sh;
      ++nb;
    });
    bad += na != nb;
  }
  return bad;
}

template <int TIER, int KIND, int D, int... Is>
int split_all(std::integer_sequence<int, Is...>) {
  return (split_mismatches<TIER, KIND, D, Is>() + ...);
}

template <int TIER>
int tier_mismatches() {
  using Seq = std::make_integer_sequence<int, 8>;
  const int split = split_all<TIER, 0, 64>(Seq{}) + split_all<TIER, 1, 64>(Seq{}) +
                    split_all<TIER, 0, 128>(Seq{}) + split_all<TIER, 1, 128>(Seq{});
  return split + mismatches<TIER, 0, 64>() + mismatches<TIER, 1, 64>() + mismatches<TIER, 0, 128>() +
         mismatches<TIER, 1, 128>();
}

int main() {
  const int bad = tier_mismatches<0>() + tier_mismatches<1>() + tier_mismatches<2>() + tier_mismatches<3>() +
                  tier_mismatches<4>() + tier_mismatches<5>();
  std::printf("layout inverse mismatches: %d\n", bad);
  return bad != 0;
}
