// Host program: prints the library's element -> (word, bit) map of a chunk (elem_pos in
// kvq_internal.cuh) for every tier, kind (0 = K, 1 = V) and D, one line per
// "tier kind D t d word bit", for comparison with the oracle's layout.
#include <cstdio>

#include "kvq_internal.cuh"

using namespace kvq;

int main() {
  for (int tier = 0; tier < kNumTiers; ++tier)
    for (int kind = 0; kind < 2; ++kind)
      for (int D : {64, 128})
        for (int t = 0; t < kPage; ++t)
          for (int d = 0; d < D; ++d) {
            int w = -1, bit = -1;
            elem_pos(kind, tier, D, t, d, w, bit);
            std::printf("%d %d %d %d %d %d %d\n", tier, kind, D, t, d, w, bit);
          }
  return 0;
}
