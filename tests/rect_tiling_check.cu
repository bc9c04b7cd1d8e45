// Host-only check of the key and query layouts the tensor-core window kernel
// loads (rect_tiling, strip_cell, rect_tiles, query_cells_per_row and
// window_query_token in area_internal.cuh).  Exit code 0 when every check
// holds; prints the failing case otherwise.  Built and run by
// tests/test_abi.py (no GPU needed).
//
// Halo rectangle of eh x ew tokens: every token must be the key of exactly
// one row of exactly one tile (the full patches first, then the strip cells,
// kCells per tile); rows outside the rectangle may only come from cells that
// stick out of its right or bottom edge, or from the unused cells of the
// last tile; when both sides are multiples of the cell's, the cell tiles
// hold a prefix of valid rows.  Window of hy x wx queries with both sides
// multiples of the cell's: positions 0 .. hy*wx-1 enumerate its tokens
// exactly once.
#include <stdio.h>

#include <vector>

#include "area_internal.cuh"

using area::kCellKeys;
using area::kCells;
using area::kCH;
using area::kCW;
using area::kPH;
using area::kPW;

static int check_rect(int eh, int ew) {
  const area::RectTiling t = area::rect_tiling(eh, ew);
  const int ntiles = area::rect_tiles(t);
  if (ntiles != t.npatch + (t.ncell + kCells - 1) / kCells) return 1;
  std::vector<int> hit(eh * ew, 0);
  const bool aligned = eh % kCH == 0 && ew % kCW == 0;
  int rows_out = 0;
  for (int jj = 0; jj < ntiles; ++jj) {
    bool seen_invalid = false;
    for (int k = 0; k < 128; ++k) {
      int y, x;
      bool exists = true;   // row holds a key of the tiling (not a padding cell)
      if (jj < t.npatch) {
        y = (jj / t.npx) * kPH + k / kPW;
        x = (jj % t.npx) * kPW + k % kPW;
      } else {
        const int c = (jj - t.npatch) * kCells + k / kCellKeys, e = k % kCellKeys;
        if (c >= t.ncell) {
          exists = false;
          y = x = 0;
        } else {
          const int2 o = area::strip_cell(t, c);
          y = o.x + e / kCW;
          x = o.y + e % kCW;
        }
      }
      const bool in = exists && y < eh && x < ew;
      if (jj < t.npatch && !in) {
        printf("rect %d x %d: patch tile %d row %d outside\n", eh, ew, jj, k);
        return 1;
      }
      if (in) {
        if (seen_invalid && aligned) {
          printf("rect %d x %d: tile %d valid row %d after an invalid one\n", eh, ew, jj, k);
          return 1;
        }
        ++hit[y * ew + x];
      } else {
        seen_invalid = true;
        ++rows_out;
      }
    }
  }
  for (int i = 0; i < eh * ew; ++i)
    if (hit[i] != 1) {
      printf("rect %d x %d: token (%d, %d) covered %d times\n", eh, ew, i / ew, i % ew, hit[i]);
      return 1;
    }
  // rows outside: at most the unused cells of the last tile plus the parts
  // of the edge cells that stick out
  const int cells_y = (eh + kCH - 1) / kCH, cells_x = (ew + kCW - 1) / kCW;
  const int bound = (kCells - 1) * kCellKeys + (cells_y * kCH) * (cells_x * kCW) - eh * ew;
  if (rows_out > bound) {
    printf("rect %d x %d: %d rows outside, bound %d\n", eh, ew, rows_out, bound);
    return 1;
  }
  return 0;
}

static int check_queries(int hy, int wx) {
  const int Wg = wx + 7;
  const int4 win = make_int4(3, 5, hy, wx);
  const int qcx = area::query_cells_per_row(win);
  const bool cells = hy % kCH == 0 && wx % kCW == 0;
  if ((qcx > 0) != cells) return 1;
  std::vector<int> hit(hy * wx, 0);
  const int nq = hy * wx;
  for (int p = 0; p < nq; ++p) {
    const int tok = area::window_query_token(win, qcx, nq, p, Wg);
    const int y = tok / Wg - win.x, x = tok % Wg - win.y;
    if (y < 0 || y >= hy || x < 0 || x >= wx) {
      printf("window %d x %d: position %d maps outside\n", hy, wx, p);
      return 1;
    }
    ++hit[y * wx + x];
  }
  for (int i = 0; i < nq; ++i)
    if (hit[i] != 1) {
      printf("window %d x %d: query (%d, %d) enumerated %d times\n", hy, wx, i / wx, i % wx, hit[i]);
      return 1;
    }
  // past the end: position 0's token
  if (area::window_query_token(win, qcx, nq, nq + 5, Wg) !=
      area::window_query_token(win, qcx, nq, 0, Wg))
    return 1;
  return 0;
}

int main() {
  int n = 0;
  for (int eh = 1; eh <= 72; ++eh)
    for (int ew = 1; ew <= 72; ++ew, ++n)
      if (check_rect(eh, ew)) return 1;
  const int big[][2] = {{200, 200}, {196, 200}, {256, 256}, {104, 52}, {393, 17}, {7, 390}};
  for (const auto& r : big) {
    ++n;
    if (check_rect(r[0], r[1])) return 1;
  }
  int nw = 0;
  for (int hy = 1; hy <= 64; ++hy)
    for (int wx = 1; wx <= 64; ++wx, ++nw)
      if (check_queries(hy, wx)) return 1;
  printf("%d rectangles and %d windows checked\n", n, nw);
  return 0;
}
