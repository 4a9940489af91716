// Host-only check of the query-block pair enumeration the 64-token path uses
// (pairs_per_group, pair_count, pair_candidates in lcsa_internal.h) and of the
// rule that picks the pairs to cut (cut_items). Built and run by
// tests/test_pair_enumeration.py; prints "ok" and exits 0 when every check
// holds, else lists the first failures and exits 1.
//
// For every block grid of 1..13 x 1..13 blocks, 1..3 frame groups and 1..2
// heads: each query block belongs to exactly one pair (a 2 x 2 group's four
// blocks counted once, through its first pair); a group's four candidates are
// a 2 x 2 square inside one frame group, listed top left, top right, bottom
// left, bottom right, and its two pairs are consecutive, slot 0 then slot 1;
// a pair outside the groups has a first row and a second row or -1.
#include <cstdio>
#include <vector>

#include "lcsa_internal.h"

int main() {
  int bad = 0, cases = 0;
  auto fail = [&](const char* what, int nHb, int nWb, long pr) {
    if (++bad <= 10) std::printf("FAIL %s: grid %d x %d, pair %ld\n", what, nHb, nWb, pr);
  };
  for (int nHb = 1; nHb <= 13; ++nHb)
    for (int nWb = 1; nWb <= 13; ++nWb)
      for (int groups = 1; groups <= 3; ++groups)
        for (int heads = 1; heads <= 2; ++heads) {
          lcsa::Grid g{};
          g.B = 1;
          g.Hn = heads;
          g.nHb = nHb;
          g.nWb = nWb;
          g.bpf = nHb * nWb;
          g.nQB = groups * g.bpf;
          const int pg = lcsa::pairs_per_group(g);
          const long np = long(lcsa::pair_count(g));
          if (np != long(heads) * groups * pg) fail("pair_count", nHb, nWb, -1);
          // a pair per two blocks, one more for an odd block count
          if (pg != (g.bpf + 1) / 2) fail("pairs_per_group", nHb, nWb, -1);
          std::vector<int> seen(size_t(heads) * g.nQB, 0);
          for (long pr = 0; pr < np; ++pr) {
            int r[4], slot;
            lcsa::pair_candidates(g, pr, r, slot);
            if (slot >= 0) {
              if (slot != int((pr % pg) & 1)) fail("slot order", nHb, nWb, pr);
              for (int i = 0; i < 4; ++i)
                if (r[i] < 0 || r[i] >= int(seen.size())) fail("row range", nHb, nWb, pr);
              if (r[1] != r[0] + 1 || r[2] != r[0] + nWb || r[3] != r[2] + 1) fail("2 x 2 square", nHb, nWb, pr);
              if (r[0] % g.bpf % nWb + 1 >= nWb || r[0] % g.bpf / nWb + 1 >= nHb) fail("inside the grid", nHb, nWb, pr);
              if (r[0] / g.bpf != r[3] / g.bpf) fail("one frame group", nHb, nWb, pr);
              if (slot == 0)
                for (int i = 0; i < 4; ++i)
                  if (r[i] >= 0 && r[i] < int(seen.size())) ++seen[r[i]];
            } else {
              if (r[0] < 0 || r[0] >= int(seen.size()) || r[1] < -1 || r[1] >= int(seen.size()))
                fail("row range", nHb, nWb, pr);
              if (r[2] != -1 || r[3] != -1) fail("unused candidates", nHb, nWb, pr);
              for (int i = 0; i < 2; ++i)
                if (r[i] >= 0 && r[i] < int(seen.size())) ++seen[r[i]];
            }
          }
          for (int v : seen)
            if (v != 1) {
              fail("each block in one pair", nHb, nWb, -1);
              break;
            }
          ++cases;
        }
  // pairs are cut only when there are at least as many as CTAs
  for (int ctas = 1; ctas <= 300; ++ctas)
    for (int items = 0; items <= 700; ++items) {
      const int c = lcsa::cut_items(items, ctas);
      if (items < ctas ? c != 0 : c != ctas / 2) fail("cut_items", items, ctas, -1);
    }
  if (bad) {
    std::printf("%d failures in %d cases\n", bad, cases);
    return 1;
  }
  std::printf("ok: %d grids\n", cases);
  return 0;
}
