// Host-only check of the persistent-grid work split used by the fused linear
// kernel (range_begin / range_owner / partial_slot / split_slot from
// fp6_linear.cuh).
// Prints "ok" or the first violated property.  Runs on the CPU.
#include <cstdio>
#include <set>
#include <vector>

#include "fp6_linear.cuh"

using namespace fp6;

static int check(long long tiles, int KT, int G) {
  const long long total = tiles * KT;
  if (G > total) G = static_cast<int>(total);
  if (range_begin(0, total, G) != 0 || range_begin(G, total, G) != total) return 1;
  for (int c = 0; c < G; ++c)
    if (range_begin(c + 1, total, G) <= range_begin(c, total, G)) return 2;  // non-empty, increasing
  int c = 0;
  for (long long i = 0; i < total; ++i) {
    while (i >= range_begin(c + 1, total, G)) ++c;
    if (range_owner(i, total, G) != c) return 3;
  }
  std::set<int> slots, counters;
  for (long long t = 0; t < tiles; ++t) {
    const int lo = range_owner(t * KT, total, G), hi = range_owner(t * KT + KT - 1, total, G);
    if (lo == hi) continue;
    if (!counters.insert(lo).second) return 4;  // counter index unique per split tile
    if (lo >= kMaxGrid) return 5;
    for (int cc = lo; cc <= hi; ++cc) {
      const int s = partial_slot(cc, t, total, G, KT);
      if (s < 0 || s >= 2 * G) return 6;
      if (split_slot(cc, lo, range_begin(lo, total, G) == t * KT) != s) return 9;   // the kernel's lookup
      if (!slots.insert(s).second) return 7;       // one slot per (CTA, split tile)
      // the CTA's segment of tile t is its first or its last segment
      const long long b = range_begin(cc, total, G), e = range_begin(cc + 1, total, G) - 1;
      if (!(b / KT == t || e / KT == t)) return 8;
    }
  }
  return 0;
}

int main() {
  const long long tiles_list[] = {1, 2, 3, 7, 56, 64, 80, 168, 224, 256, 448, 1000, 3584};
  const int kt_list[] = {1, 2, 8, 112, 128, 448};
  const int g_list[] = {1, 2, 3, 16, 132, 148, 160};
  for (long long t : tiles_list)
    for (int kt : kt_list)
      for (int g : g_list) {
        const int r = check(t, kt, g);
        if (r) {
          std::printf("fail %d tiles=%lld KT=%d G=%d\n", r, t, kt, g);
          return 1;
        }
      }
  std::printf("ok\n");
  return 0;
}
