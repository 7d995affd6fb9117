// Host-only check of the attention work split (cta_begin / cta_of_step in gca_internal.h), the
// bookkeeping that the attention kernel, the combine kernel and the host planner share. For many
// shapes (key tiles per unit, units, CTAs, cost of a move to another unit) it checks that:
//   - the CTA ranges start at 0, end at total and never go backwards;
//   - cta_of_step(s) is the last CTA c with cta_begin(c) <= s, by brute force over all steps;
//   - the partial-record slots 2*(c + u2) + q of all (CTA, unit) pieces are distinct and below
//     2*(grid + units2) (the size the scratch and the no-allocation array are planned for);
//   - with the cost charged (16 <= total/grid steps, as the planner applies it) no range is
//     empty, and CTAs that move to another unit get no more steps than those that do not, less
//     the charge.
// Prints "ok <shapes>" and exits 0, or prints the first failure and exits 1. No GPU is used.
#include <cstdio>
#include <cstring>
#include <set>
#include <vector>

#include "gca_internal.h"

namespace {

int fail(const char* what, int n_tiles, int units2, int grid, int gap, long long a, long long b) {
  std::printf("FAIL %s: n_tiles %d units2 %d grid %d gap %d (%lld, %lld)\n", what, n_tiles, units2,
              grid, gap, a, b);
  return 1;
}

int check(int n_tiles, int units2, int grid, int gap) {
  gca::AttnParams p;
  std::memset(&p, 0, sizeof(p));
  p.n_tiles = n_tiles;
  p.units2 = units2;
  p.grid = grid;
  p.unit_gap = gap;
  const long long total = (long long)n_tiles * units2;
  p.total = total;
  std::vector<long long> b(grid + 1);
  for (int c = 0; c <= grid; ++c) b[c] = gca::cta_begin(c, p);
  if (b[0] != 0 || b[grid] != total) return fail("ends", n_tiles, units2, grid, gap, b[0], b[grid]);
  for (int c = 0; c < grid; ++c) {
    if (b[c + 1] < b[c]) return fail("monotone", n_tiles, units2, grid, gap, c, b[c]);
  }
  // brute-force inverse
  int c = 0;
  for (long long s = 0; s < total; ++s) {
    while (c + 1 < grid && b[c + 1] <= s) ++c;
    const long long got = gca::cta_of_step(s, p);
    if (got != c) return fail("cta_of_step", n_tiles, units2, grid, gap, s, got);
  }
  // partial slots of every (CTA, unit) piece
  std::set<long long> slots;
  for (int cc = 0; cc < grid; ++cc) {
    if (b[cc] == b[cc + 1]) continue;
    const long long u0 = b[cc] / n_tiles, u1 = (b[cc + 1] - 1) / n_tiles;
    for (long long u = u0; u <= u1; ++u) {
      for (int q = 0; q < gca::kQPerCta; ++q) {
        const long long sl = gca::part_slot(cc, u, q);
        if (sl < 0 || sl >= 2LL * (grid + units2)) {
          return fail("slot range", n_tiles, units2, grid, gap, cc, sl);
        }
        if (!slots.insert(sl).second) return fail("slot reuse", n_tiles, units2, grid, gap, cc, sl);
      }
    }
  }
  if (gap > 0 && total >= 16LL * grid) {
    long long max_one = 0, min_one = total + 1, max_moving = 0;
    for (int cc = 0; cc < grid; ++cc) {
      const long long len = b[cc + 1] - b[cc];
      if (len == 0) return fail("empty range", n_tiles, units2, grid, gap, cc, 0);
      const bool moves = b[cc] / n_tiles != (b[cc + 1] - 1) / n_tiles;
      if (moves) {
        if (len > max_moving) max_moving = len;
      } else {
        if (len > max_one) max_one = len;
        if (len < min_one) min_one = len;
      }
    }
    // a CTA that moves pays the charge: it never holds more steps than a CTA that stays in one
    // unit holds at most, less the charge, plus the one step of rounding either side
    if (max_moving > 0 && min_one <= total && max_moving > max_one - gap + 2) {
      return fail("charge", n_tiles, units2, grid, gap, max_moving, max_one);
    }
  }
  return 0;
}

}  // namespace

int main() {
  const int tiles[] = {1, 2, 5, 11, 17, 50, 96, 189, 217, 700};
  const int units[] = {1, 2, 3, 16, 64, 256};
  const int grids[] = {1, 2, 7, 64, 148, 512};
  const int gaps[] = {0, 1, 4, 6};
  int shapes = 0;
  for (int t : tiles) {
    for (int u : units) {
      for (int g : grids) {
        for (int gap : gaps) {
          if ((long long)t * u > 200000) continue;
          if (check(t, u, g, gap)) return 1;
          ++shapes;
        }
      }
    }
  }
  std::printf("ok %d shapes\n", shapes);
  return 0;
}
