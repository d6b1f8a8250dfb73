// Work schedule of the persistent Hessian kernel (host and device).
//
// Output tiles are 128 rows (i) x 256 columns (j) of H; only tiles touching the upper
// triangle exist (row block bi, column block bj with bi*128 <= bj*256 + 255).
//
// Tile order: super-blocks of 16 x 8 tiles (2048 x 2048 channels), walked by super-column;
// inside a super-column the off-diagonal super-blocks come first (rows outer), then the
// diagonal one.  Consecutive tiles therefore share their channels, and any wave of G
// consecutive tiles reads about 4-5 K distinct channels instead of nearly all of them.
//
// Units: (tile, token segment) with S segments per tile.  The tile list is cut into
// groups of G (the grid size); group k's units are numbered segment-major, so that wave w
// (units w*G .. w*G+G-1) processes one token segment of one group: all CTAs read the same
// token rows at about the same time and the rows stay in L2 between their readers.  CTA c
// takes units c, c+G, c+2G, ...: inside a full group that is one tile over all S segments
// in a row (accumulated without any intermediate write-back); only the last, partial group
// spreads its tiles' segments over every CTA.
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define HSCHED_FN __host__ __device__ __forceinline__
#else
#define HSCHED_FN inline
#endif

namespace gptq {
namespace hsched {

constexpr int TM = 128, TN = 256;  // tile rows, tile columns
constexpr int SR = 16, SC = 8;     // tiles per super-block: rows, columns

HSCHED_FN int row_blocks(int n) { return (n + TM - 1) / TM; }
HSCHED_FN int col_blocks(int n) { return (n + TN - 1) / TN; }

HSCHED_FN int tile_count(int n) {
  const int rb = row_blocks(n), cb = col_blocks(n);
  int t = 0;
  for (int j = 0; j < cb; ++j) t += rb < 2 * j + 2 ? rb : 2 * j + 2;
  return t;
}

// Tile t (0 <= t < tile_count(n)) in super-block order.
HSCHED_FN void tile_at(int t, int n, int& bi, int& bj) {
  const int rb = row_blocks(n), cb = col_blocks(n);
  for (int sj = 0; sj * SC < cb; ++sj) {
    const int nc = cb - sj * SC < SC ? cb - sj * SC : SC;  // columns of this super-column
    const int nr = rb - sj * SR < SR ? rb - sj * SR : SR;  // rows of its diagonal block
    const int off = sj * SR * nc;                          // off-diagonal tiles (all rows valid)
    if (t < off) {
      const int si = t / (SR * nc), rem = t % (SR * nc);
      bi = si * SR + rem / nc;
      bj = sj * SC + rem % nc;
      return;
    }
    t -= off;
    for (int c = 0; c < nc; ++c) {  // diagonal block: rows r <= 2c + 1
      const int k = nr < 2 * c + 2 ? nr : 2 * c + 2;
      if (t < k) {
        bi = sj * SR + t;
        bj = sj * SC + c;
        return;
      }
      t -= k;
    }
  }
  bi = 0;
  bj = 0;
}

// Unit u (0 <= u < tiles * S < 2^31) -> (tile index, token segment).
HSCHED_FN void unit_at(int u, int tiles, int S, int G, int& tile, int& seg) {
  const int full = tiles / G;  // full groups
  const int per_group = G * S;
  if (u < full * per_group) {
    const int k = u / per_group, rem = u % per_group;
    seg = rem / G;
    tile = k * G + rem % G;
  } else {
    const int g = tiles - full * G;  // tiles of the last, partial group
    const int rem = u - full * per_group;
    seg = rem / g;
    tile = full * G + rem % g;
  }
}

}  // namespace hsched
}  // namespace gptq
