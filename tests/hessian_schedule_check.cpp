// Host check of the persistent Hessian kernel's work schedule (csrc/hessian_sched.cuh):
// tile_at enumerates exactly the tiles that touch the upper triangle, and unit_at covers
// every (tile, token segment) exactly once, for many orders and grid / segment counts.
// Exits nonzero on the first mismatch.
#include <cstdio>
#include <set>
#include <utility>

#include "hessian_sched.cuh"

using namespace gptq::hsched;

int main() {
  int bad = 0;
  for (int n = 8; n <= 20000; n += (n < 600 ? 8 : 1000 + 8)) {
    const int rb = row_blocks(n), cb = col_blocks(n), tiles = tile_count(n);
    std::set<std::pair<int, int>> want, got;
    for (int j = 0; j < cb; ++j)
      for (int i = 0; i < rb && i * TM <= j * TN + TN - 1; ++i) want.insert({i, j});
    for (int t = 0; t < tiles; ++t) {
      int bi, bj;
      tile_at(t, n, bi, bj);
      got.insert({bi, bj});
    }
    if (want != got || static_cast<int>(got.size()) != tiles) {
      std::printf("tile set mismatch at n=%d\n", n);
      ++bad;
    }
    for (int G : {1, 7, 148, 296}) {
      for (int S : {1, 3, 7}) {
        if (G > tiles * S) continue;
        std::set<std::pair<int, int>> units;
        for (int u = 0; u < tiles * S; ++u) {
          int tile, seg;
          unit_at(u, tiles, S, G, tile, seg);
          if (tile < 0 || tile >= tiles || seg < 0 || seg >= S) {
            std::printf("unit out of range at n=%d G=%d S=%d u=%d\n", n, G, S, u);
            ++bad;
            break;
          }
          units.insert({tile, seg});
        }
        if (static_cast<long>(units.size()) != static_cast<long>(tiles) * S) {
          std::printf("units do not cover (tile, segment) at n=%d G=%d S=%d\n", n, G, S);
          ++bad;
        }
      }
    }
  }
  std::printf(bad ? "FAILED %d\n" : "ok\n", bad);
  return bad != 0;
}
