// Recursion plan of the damped inverse-Cholesky factor (host code, shared by factor.cu and a
// host test): where each block splits, which nodes form their products on the int8 tensor
// cores, and the largest scratch each recursion depth needs.
//
// Block [lo, hi) of order n splits at hi - n2 with n2 = ceil(n/2) rounded up to a multiple of
// NB (the larger part bottom right); blocks of at most NB are leaves.  A node whose right part
// is at least I8_MIN wide forms its four products from int8 operand slices (both K of its
// products, n2 and n1 <= n2, stay within the int8 kernel's 16384); smaller ones use the fp64
// matrix units.
#pragma once

#include <algorithm>
#include <cstddef>
#include <cstdint>
#include <vector>

namespace gptq {
namespace fplan {

constexpr int NB = 128;  // leaf block width of the factorisation
constexpr int64_t I8_MIN = 1024;
constexpr int64_t I8_MAX = 16384;

inline int64_t right_part(int64_t n) {
  const int64_t half = (n + 1) / 2;
  return std::min<int64_t>(n - 1, ((half + NB - 1) / NB) * NB);
}

inline bool node_i8(int64_t n2) { return n2 >= I8_MIN && n2 <= I8_MAX; }

inline int64_t pad64(int64_t k) { return (k + 63) / 64 * 64; }

struct Plan {
  size_t pmax = 0;
  std::vector<size_t> tmax;            // T per depth
  std::vector<size_t> sx, sy, ex, ey;  // int8 slices (bytes) and exponents per depth
};

// Largest P (n1 x n2) over all nodes, and per recursion depth the largest T and int8 slice
// buffers for `ks` slices: X [ks][n1][pad(n2)] (rows of B, then of P, then of U11),
// Y [ks][n2][pad(n2)] (rows of U22, then its columns, then the columns of T).
inline void plan(int64_t n, int depth, Plan& pl, size_t ks) {
  if (n <= NB) return;
  const int64_t n2 = right_part(n), n1 = n - n2;
  const size_t sz = static_cast<size_t>(n1) * n2;
  pl.pmax = std::max(pl.pmax, sz);
  const size_t d = static_cast<size_t>(depth);
  for (auto* v : {&pl.tmax, &pl.sx, &pl.sy, &pl.ex, &pl.ey})
    if (v->size() <= d) v->resize(d + 1, 0);
  pl.tmax[d] = std::max(pl.tmax[d], sz);
  if (node_i8(n2)) {
    pl.sx[d] = std::max(pl.sx[d], ks * n1 * pad64(n2));
    pl.sy[d] = std::max(pl.sy[d], ks * n2 * pad64(n2));
    pl.ex[d] = std::max(pl.ex[d], static_cast<size_t>(n1));
    pl.ey[d] = std::max(pl.ey[d], static_cast<size_t>(n2));
  }
  plan(n2, depth + 1, pl, ks);
  plan(n1, depth + 1, pl, ks);
}

}  // namespace fplan
}  // namespace gptq
