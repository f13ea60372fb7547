// Host-side check of the few-token kernel's stream-K work split, compiled
// with nvcc against the kernel's own header and run on the CPU (no GPU
// call). For every (units, grid, kc) tried it checks that
//   * the CTA ranges [begin(c), begin(c+1)) tile [0, units) in order, and
//     every CTA gets at least floor(units / grid) units;
//   * smallm_cta_of(u) is the CTA whose range holds u;
//   * a band of kc consecutive units is shared by the CTAs
//     cta_of(first) .. cta_of(last), the count the kernel's last-arriver
//     rule uses, and each CTA parks at most two pieces: the band its range
//     starts in (when an earlier CTA started it) and the band it ends in
//     (when a later CTA finishes it), never the same band twice.
// Prints "ok" and exits 0, or prints the first violation and exits 1.
#include <cstdio>
#include <vector>

#include "smallm.cuh"

using qlora::smallm_cta_of;
using qlora::smallm_unit_begin;

static int fail(const char *what, long units, long grid, long kc, long x) {
  std::printf("FAIL %s: units %ld grid %ld kc %ld at %ld\n", what, units, grid, kc, x);
  return 1;
}

int main() {
  const long kcs[] = {1, 2, 3, 4, 16, 32, 43, 86};
  for (long kc : kcs) {
    for (long bands = 1; bands <= 90; bands += (bands < 20 ? 1 : 7)) {
      const long units = bands * kc;
      for (long grid = 1; grid <= 148; ++grid) {
        if (grid > units) break;
        // ranges tile [0, units)
        if (smallm_unit_begin(0, units, grid) != 0) return fail("begin(0)", units, grid, kc, 0);
        if (smallm_unit_begin(grid, units, grid) != units) return fail("begin(grid)", units, grid, kc, grid);
        for (long c = 0; c < grid; ++c) {
          const long b0 = smallm_unit_begin(c, units, grid), b1 = smallm_unit_begin(c + 1, units, grid);
          if (b1 - b0 < units / grid) return fail("range size", units, grid, kc, c);
          for (long u = b0; u < b1; ++u)
            if (smallm_cta_of(u, units, grid) != c) return fail("cta_of", units, grid, kc, u);
        }
        // pieces per band, and at most two parked pieces per CTA
        std::vector<int> parked(grid, 0), first_b(grid, -1), last_b(grid, -1);
        for (long b = 0; b < bands; ++b) {
          const long f = b * kc, l = f + kc - 1;
          const long c0 = smallm_cta_of(f, units, grid), c1 = smallm_cta_of(l, units, grid);
          long sharing = 0;
          for (long c = 0; c < grid; ++c) {
            const long b0 = smallm_unit_begin(c, units, grid), b1 = smallm_unit_begin(c + 1, units, grid);
            if (b0 <= l && b1 > f) ++sharing;
          }
          if (sharing != c1 - c0 + 1) return fail("pieces", units, grid, kc, b);
          if (c0 == c1) continue;  // a whole band on one CTA: finished there, nothing parked
          for (long c = c0; c <= c1; ++c) {
            const long b0 = smallm_unit_begin(c, units, grid);
            // slot 1: the CTA starts the band (its range holds the band's first unit);
            // slot 0: a later piece of a band an earlier CTA started
            int &slot = (b0 <= f) ? last_b[c] : first_b[c];
            if (slot >= 0) return fail("slot reused", units, grid, kc, c);
            slot = static_cast<int>(b);
            ++parked[c];
          }
        }
        for (long c = 0; c < grid; ++c)
          if (parked[c] > 2) return fail("more than two pieces", units, grid, kc, c);
      }
    }
  }
  std::printf("ok\n");
  return 0;
}
