// Host-only check of the merge geometry the window kernels use (axis_merge,
// merge_role, axis_twice_total in area_internal.cuh), over every token of a
// set of tilings.  Exit code 0 when every check holds; prints the failing
// case otherwise.  Built and run by tests/test_abi.py (no GPU needed).
#include <stdio.h>
#include <stdlib.h>

#include <vector>

#include "area_internal.cuh"

using area::axis_merge;
using area::axis_twice_total;
using area::axis_window;
using area::merge_role;
using area::MergeRole;

static int check(int Hg, int Wg, int w, int sy, int sx) {
  const int hy = w < Hg ? w : Hg, wx = w < Wg ? w : Wg;
  const int nby = (Hg + sy + hy - 1) / hy, nbx = (Wg + sx + wx - 1) / wx;
  const int ny2 = axis_twice_total(nby, Hg, hy, sy), nx2 = axis_twice_total(nbx, Wg, wx, sx);
  const long long n_ov = (long long)ny2 * Wg + (long long)(Hg - ny2) * nx2;
  const int N = Hg * Wg;
  std::vector<int> cover(N, 0), firsts(N, 0), lasts(N, 0), classes(N, 0);
  std::vector<long long> rank(N, -1);
  for (int iy = 0; iy < nby; ++iy) {
    int y0, h;
    axis_window(iy, nby, Hg, hy, sy, &y0, &h);
    const int4 my = axis_merge(iy, nby, Hg, hy, sy);
    for (int ix = 0; ix < nbx; ++ix) {
      int x0, wd;
      axis_window(ix, nbx, Wg, wx, sx, &x0, &wd);
      const int4 mx = axis_merge(ix, nbx, Wg, wx, sx);
      const int cls = ((iy & 1) << 1) | (ix & 1);
      if (my.x != y0 || mx.x != x0) {
        printf("window start mismatch Hg=%d Wg=%d w=%d s=(%d,%d)\n", Hg, Wg, w, sy, sx);
        return 1;
      }
      for (int y = y0; y < y0 + h; ++y)
        for (int x = x0; x < x0 + wd; ++x) {
          const int t = y * Wg + x;
          const MergeRole r = merge_role(y, x, cls, my, mx, Wg, nx2);
          ++cover[t];
          if (classes[t] & (1 << cls)) {
            printf("two windows of class %d share token %d\n", cls, t);
            return 1;
          }
          classes[t] |= 1 << cls;
          firsts[t] += r.first;
          lasts[t] += r.last;
          if (r.ov) {
            if (rank[t] >= 0 && rank[t] != r.rank) {
              printf("windows disagree on the row of token %d\n", t);
              return 1;
            }
            rank[t] = r.rank;
          } else if (!(r.first && r.last)) {
            printf("single-window token %d is not first and last\n", t);
            return 1;
          }
        }
    }
  }
  long long next = 0;
  for (int t = 0; t < N; ++t) {
    if (cover[t] < 1 || cover[t] > 4) {
      printf("token %d covered %d times (Hg=%d Wg=%d w=%d s=(%d,%d))\n", t, cover[t], Hg, Wg, w,
             sy, sx);
      return 1;
    }
    if (firsts[t] != 1 || lasts[t] != 1) {
      printf("token %d: %d first and %d last windows\n", t, firsts[t], lasts[t]);
      return 1;
    }
    const bool ov = cover[t] > 1;
    if (ov != (rank[t] >= 0)) {
      printf("token %d: overlap flag disagrees with cover %d\n", t, cover[t]);
      return 1;
    }
    if (ov && rank[t] != next++) {   // rows numbered in token order, no gap
      printf("token %d: row %lld, expected %lld (Hg=%d Wg=%d w=%d s=(%d,%d))\n", t, rank[t],
             next - 1, Hg, Wg, w, sy, sx);
      return 1;
    }
  }
  if (next != n_ov) {
    printf("n_ov %lld but %lld overlapped tokens\n", n_ov, next);
    return 1;
  }
  return 0;
}

int main() {
  int cases = 0;
  // the configurations' grids and schedules
  const int grids[][2] = {{32, 32}, {128, 128}, {256, 256}, {384, 384}, {384, 128}};
  const int sides[] = {8, 20, 32, 40, 48, 56, 64, 72, 80, 88, 96, 104, 112, 120, 144, 168,
                       176, 192, 208, 224, 256, 272};
  for (auto& g : grids)
    for (int w : sides) {
      if (check(g[0], g[1], w, 0, 0)) return 1;
      ++cases;
    }
  // small grids, every window side and border shift
  for (int Hg = 2; Hg <= 30; Hg += 2)
    for (int Wg = 2; Wg <= 26; Wg += 4)
      for (int w = 1; w <= 24; ++w) {
        const int hy = w < Hg ? w : Hg, wx = w < Wg ? w : Wg;
        for (int sy = 0; sy < (hy < Hg ? hy : 1); ++sy)
          for (int sx = 0; sx < (wx < Wg ? wx : 1); sx += 3) {
            if (check(Hg, Wg, w, sy, sx)) return 1;
            ++cases;
          }
      }
  printf("merge geometry: %d tilings checked\n", cases);
  return 0;
}
