// Host check of the factor's recursion plan (csrc/factor_plan.h): for many orders, every node
// of the recursion fits the scratch that the plan reserves for its depth (P, T, and for int8
// nodes both slice buffers in each of their uses and the exponent arrays), every int8 node
// stays within the int8 kernel's K limit with K padded to 64, and the split is the documented
// one (n2 a multiple of NB unless the block is only one wider than NB, n1 <= n2).
// Exits nonzero on the first violation.
#include <cstdio>

#include "factor_plan.h"

using namespace gptq::fplan;

static int bad = 0;

static void check_node(int64_t m, int depth, const Plan& pl, size_t ks, int64_t n, int64_t* i8_nodes) {
  if (m <= NB) return;
  const int64_t n2 = right_part(m), n1 = m - n2;
  const size_t d = static_cast<size_t>(depth);
  auto fail = [&](const char* what) {
    if (bad < 20) std::printf("n=%lld node m=%lld depth=%d: %s\n", (long long)n, (long long)m, depth, what);
    ++bad;
  };
  if (n1 < 1 || n2 < 1 || n1 > n2) fail("split sizes");
  if (n2 % NB != 0 && n2 != m - 1) fail("n2 not a multiple of NB");
  if (d >= pl.tmax.size()) {
    fail("depth beyond the plan");
    return;
  }
  const size_t sz = static_cast<size_t>(n1) * n2;
  if (sz > pl.pmax || sz > pl.tmax[d]) fail("P or T too small");
  if (node_i8(n2)) {
    ++*i8_nodes;
    const size_t k2 = static_cast<size_t>(pad64(n2)), k1 = static_cast<size_t>(pad64(n1));
    if (k2 % 64 || k1 % 64 || k2 > static_cast<size_t>(I8_MAX) || k1 > static_cast<size_t>(I8_MAX))
      fail("padded K outside the int8 kernel's range");
    // X: rows of B and of P ([ks][n1][k2]), then rows of U11 ([ks][n1][k1]);
    // Y: rows and columns of U22 ([ks][n2][k2]), then columns of T ([ks][n2][k1])
    if (ks * n1 * k2 > pl.sx[d] || ks * n1 * k1 > pl.sx[d]) fail("X slices too small");
    if (ks * n2 * k2 > pl.sy[d] || ks * n2 * k1 > pl.sy[d]) fail("Y slices too small");
    if (static_cast<size_t>(n1) > pl.ex[d] || static_cast<size_t>(n2) > pl.ey[d]) fail("exponents too small");
  } else if (n2 >= I8_MIN && n2 <= I8_MAX) {
    fail("node in the int8 range not taken");
  }
  check_node(n2, depth + 1, pl, ks, n, i8_nodes);
  check_node(n1, depth + 1, pl, ks, n, i8_nodes);
}

int main() {
  const size_t ks = 7;
  int64_t total_i8 = 0;
  for (int64_t n = 8; n <= 65535; n += (n < 3000 ? 8 : 997)) {
    Plan pl;
    plan(n, 0, pl, ks);
    int64_t i8 = 0;
    check_node(n, 0, pl, ks, n, &i8);
    total_i8 += i8;
  }
  for (int64_t n : {4096, 8192, 11008, 14336, 28672, 65528}) {
    Plan pl;
    plan(n, 0, pl, ks);
    int64_t i8 = 0;
    check_node(n, 0, pl, ks, n, &i8);
    total_i8 += i8;
  }
  // the Llama-2-7B layer's orders: 4096 has int8 nodes at depths 0-1 (3 nodes), 11008 at 0-2
  // (7 nodes); the first order with one is 1793 (its right part rounds up to 1024)
  for (auto [n, want] : {std::pair<int64_t, int64_t>{4096, 3}, {11008, 7}, {1793, 1}, {1792, 0}}) {
    Plan pl;
    plan(n, 0, pl, ks);
    int64_t i8 = 0;
    check_node(n, 0, pl, ks, n, &i8);
    if (i8 != want) {
      std::printf("n=%lld: %lld int8 nodes, expected %lld\n", (long long)n, (long long)i8, (long long)want);
      ++bad;
    }
  }
  if (bad) {
    std::printf("%d violations\n", bad);
    return 1;
  }
  std::printf("checked (%lld int8 nodes) ok\n", (long long)total_i8);
  return 0;
}
