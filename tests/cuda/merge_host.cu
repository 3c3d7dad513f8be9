// Host-side check of the attention kernel's merged tile order (Merge in
// ab_attention.cuh) for every pair of stream lengths T0, T1 <= 96: tile() and
// index() are inverse bijections between [0, T0 + T1) and the (stream, tile)
// pairs, each stream's tiles come in increasing order, and the two streams
// alternate (0, 1, 0, 1, ...) for as long as both have tiles.
// Exits 1 on any violation.
#include <cstdio>
#include <vector>

#include "ab_attention.cuh"

int main() {
  long bad = 0, cases = 0;
  for (int T0 = 0; T0 <= 96; ++T0) {
    for (int T1 = 0; T1 <= 96; ++T1) {
      const ab::Merge mg(T0, T1);
      if (mg.total() != T0 + T1) ++bad;
      std::vector<int> seen0(T0, 0), seen1(T1, 0);
      int last[2] = {-1, -1};
      const int m = T0 < T1 ? T0 : T1;
      for (int g = 0; g < mg.total(); ++g) {
        int s = -1, t = -1;
        mg.tile(g, s, t);
        ++cases;
        const int T = s == 0 ? T0 : T1;
        if ((s != 0 && s != 1) || t < 0 || t >= T) { ++bad; continue; }
        (s == 0 ? seen0 : seen1)[t] += 1;
        if (mg.index(s, t) != g) ++bad;
        if (t != last[s] + 1) ++bad;  // in order, no gaps
        last[s] = t;
        if (g < 2 * m && s != (g & 1)) ++bad;  // alternation while both streams have tiles
      }
      for (int v : seen0) bad += v != 1;
      for (int v : seen1) bad += v != 1;
    }
  }
  std::printf("cases %ld violations %ld\n", cases, bad);
  return bad ? 1 : 0;
}
