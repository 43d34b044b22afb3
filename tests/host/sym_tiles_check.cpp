// Host check of the symmetric-product tiling of the tensor-core path
// (for_each_sym_tile, split_n and sym_block_mode, the functions the kernel
// and the plan use).
//
// For every m in [1, 2100], and for the tiles split along N 0, 1 and 2 times:
//  - every tile has 1 <= n_need <= 256 columns, rows and staged B rows that
//    start on a multiple of 16 elements (TMA alignment), and a contiguous
//    tile's second half starts where its first ends;
//  - walking each CTA's 32-row groups and each 32-column chunk of the
//    accumulator exactly as the epilogue does, the blocks that
//    sym_block_mode writes cover each element (i, j), j <= i, of the lower
//    triangle exactly once (a block written with its mirror covers (i, j)
//    for all its elements, a diagonal block the elements with j <= i).
// Prints "ok <tiles for m = 1408> <tiles for m = 2048>" (unsplit), then
// "split <level> <tiles for m = 1408> <tiles for m = 2048>" per level, or the
// first violation.
#include "muon_internal.cuh"

#include <cstdio>
#include <vector>

int main() {
  using namespace muon;
  for (int level = 0; level <= 2; ++level) {
  int tiles_1408 = 0, tiles_2048 = 0;
  for (int m = 1; m <= 2100; ++m) {
    std::vector<unsigned char> cover(static_cast<size_t>(m) * m, 0);
    bool bad = false;
    int count = 0;
    for_each_sym_tile(m, [&](const TcTile& whole) { split_n(whole, level, m, [&](const TcTile& t) {
      ++count;
      const int n_mma = tile_n_mma(t.n_need), half = n_mma / 2;
      if (t.n_need < 1 || t.n_need > 256 || t.r0 % 16 || t.r1 % 16 || t.c0 % 16 || t.c1 % 16 || t.r0 >= m ||
          t.c0 >= m) {
        std::printf("m=%d: tile (%d %d | %d %d, %d) malformed\n", m, t.r0, t.r1, t.c0, t.c1, t.n_need);
        bad = true;
        return;
      }
      for (int rank = 0; rank < 2 && !bad; ++rank) {
        const int rbase = rank ? t.r1 : t.r0;
        for (int q4 = 0; q4 < 4 && !bad; ++q4) {
          const int i_lo = rbase + 32 * q4;
          for (int cc = 0; cc < t.n_need && !bad; cc += 32) {
            const int j0 = cc < half ? t.c0 + cc : t.c1 + (cc - half);
            const int md = sym_block_mode(t.flags, rank, i_lo, j0);
            if (md == 0) continue;
            for (int i = i_lo; i < i_lo + 32 && i < m; ++i)
              for (int j = j0; j < j0 + 32 && j < m; ++j) {
                if (md == 2 && j > i) continue;
                const int r = i >= j ? i : j, c = i >= j ? j : i;
                if (md == 1 && j > i) {
                  std::printf("m=%d: block (%d, %d) above the diagonal written whole\n", m, i_lo, j0);
                  bad = true;
                  return;
                }
                if (++cover[static_cast<size_t>(r) * m + c] > 1) {
                  std::printf("m=%d: element (%d, %d) written twice\n", m, r, c);
                  bad = true;
                  return;
                }
              }
          }
        }
      }
    }); });
    for (int r = 0; r < m && !bad; ++r)
      for (int c = 0; c <= r; ++c)
        if (cover[static_cast<size_t>(r) * m + c] != 1) {
          std::printf("m=%d: element (%d, %d) not covered\n", m, r, c);
          bad = true;
          break;
        }
    if (bad) return 1;
    if (m == 1408) tiles_1408 = count;
    if (m == 2048) tiles_2048 = count;
  }
  if (level == 0) std::printf("ok %d %d\n", tiles_1408, tiles_2048);
  else std::printf("split %d %d %d\n", level, tiles_1408, tiles_2048);
  }
  // The X-update tiles (for_each_full_tile), split 0, 1 and 2 times: walking
  // each CTA's 128 rows and the accumulator's 32-column chunks as the
  // epilogue does (rows and columns past the product masked), every element
  // of the R x C output is written exactly once.
  for (int level = 0; level <= 2; ++level) {
    for (int R = 1; R <= 700; R += 23)
      for (int C = 1; C <= 1100; C += 37) {
        std::vector<unsigned char> cover(static_cast<size_t>(R) * C, 0);
        bool bad = false;
        for_each_full_tile(R, C, [&](const TcTile& whole) { split_n(whole, level, C, [&](const TcTile& t) {
          const int half = tile_n_mma(t.n_need) / 2;
          if (t.n_need < 1 || t.n_need > 256 || t.c0 % 16 || t.c1 % 16 || t.c0 >= C) {
            std::printf("R=%d C=%d: tile (%d %d | %d %d, %d) malformed\n", R, C, t.r0, t.r1, t.c0, t.c1, t.n_need);
            bad = true;
            return;
          }
          for (int rank = 0; rank < 2; ++rank)
            for (int i = rank ? t.r1 : t.r0, e = i + 128; i < e && i < R; ++i)
              for (int cc = 0; cc < t.n_need; ++cc) {
                const int j = cc < half ? t.c0 + cc : t.c1 + (cc - half);
                if (j < C && ++cover[static_cast<size_t>(i) * C + j] > 1) bad = true;
              }
        }); });
        for (size_t k = 0; k < cover.size() && !bad; ++k)
          if (cover[k] != 1) bad = true;
        if (bad) {
          std::printf("full tiles R=%d C=%d split %d: an element not written exactly once\n", R, C, level);
          return 1;
        }
      }
  }
  std::printf("full ok\n");
  return 0;
}
