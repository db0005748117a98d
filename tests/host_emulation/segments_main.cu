// Host check of the LSA scan's list-segment arithmetic (lsa_first_cta,
// lsa_segment, lsa_max_segments in kernels.h, shared by the scan kernel, the
// compaction kernel and the workspace sizing).  For every (T, P, cap2)
// given on the command line: each query group's segments, one per CTA that
// scores the group, must tile [0, cap2 + slack * covering CTAs) in CTA order
// without gaps or overlaps, index the counters below nseg, and fit the row
// width the host reserves.  Prints "ok" or the first violation.  Test
// infrastructure only.
#include <cstdio>
#include <cstdlib>
#include "kernels.h"

using namespace lsi;

static int check(int T, int P, int cap2, int grid_cap) {
  const int QB = 256, BM = 128, slack = 64;
  const int NT = (P + BM - 1) / BM, G = (T + QB - 1) / QB;
  const long long units = static_cast<long long>(G) * NT;
  const int grid = static_cast<int>(units < grid_cap ? units : grid_cap);
  const int nseg = lsa_max_segments(units, grid, NT);
  const long long per_row = cap2 + static_cast<long long>(slack) * nseg;
  for (int g = 0; g < G; ++g) {
    const int c0 = lsa_first_cta(units, grid, NT, g);
    long long expect_off = 0;
    int covering = 0;
    for (int c = 0; c < grid; ++c) {
      const long long ub = units * c / grid, ue = units * (c + 1) / grid;
      const bool covers = (ub > static_cast<long long>(g) * NT ? ub : static_cast<long long>(g) * NT) <
                          (ue < static_cast<long long>(g + 1) * NT ? ue : static_cast<long long>(g + 1) * NT);
      const LsaSeg s = lsa_segment(units, grid, NT, g, c, cap2, slack);
      if (!covers) {
        if (s.len != 0) { std::printf("T=%d P=%d g=%d c=%d: len %d for a CTA that does not score the group\n", T, P, g, c, s.len); return 1; }
        continue;
      }
      if (s.j != c - c0 || s.j < 0 || s.j >= nseg) { std::printf("T=%d P=%d g=%d c=%d: j=%d (first %d, nseg %d)\n", T, P, g, c, s.j, c0, nseg); return 1; }
      if (s.off != expect_off || s.len <= 0) { std::printf("T=%d P=%d g=%d c=%d: off %lld (want %lld) len %d\n", T, P, g, c, static_cast<long long>(s.off), expect_off, s.len); return 1; }
      expect_off = s.off + s.len;
      ++covering;
    }
    if (covering == 0 || expect_off != cap2 + static_cast<long long>(slack) * covering || expect_off > per_row) {
      std::printf("T=%d P=%d g=%d: segments end at %lld for %d CTAs (row width %lld)\n", T, P, g, expect_off, covering, per_row);
      return 1;
    }
  }
  return 0;
}

int main(int argc, char** argv) {
  int bad = 0;
  for (int i = 1; i + 3 < argc + 1 && i + 3 <= argc; i += 4)
    bad |= check(std::atoi(argv[i]), std::atoi(argv[i + 1]), std::atoi(argv[i + 2]), std::atoi(argv[i + 3]));
  std::printf(bad ? "FAIL\n" : "ok\n");
  return bad;
}
