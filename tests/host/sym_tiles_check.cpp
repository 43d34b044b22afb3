// Host check of the symmetric-product tile list (for_each_sym_tile).
//
// For every m in [1, 2100] the list must:
//  - put every tile on the 256 x 256 grid with 1 <= need <= 256 columns
//    inside the matrix;
//  - have full rows (row0 + 256 <= m) in every tile whose rows are not the
//    diagonal block of the last, ragged row block;
//  - cover each element (i, j), j <= i, of the lower triangle exactly once,
//    counting a transposed tile (col0 > row0) by its mirror.
// Prints "ok <tiles for m = 1408>" or the first violation.
#include "muon_internal.cuh"

#include <cstdio>
#include <vector>

int main() {
  using muon::kTileM;
  int tiles_1408 = 0;
  for (int m = 1; m <= 2100; ++m) {
    std::vector<unsigned char> cover(static_cast<size_t>(m) * m, 0);
    bool bad = false;
    int count = 0;
    muon::for_each_sym_tile(m, [&](int row0, int col0, int need) {
      ++count;
      if (row0 % kTileM || col0 % kTileM || need < 1 || need > kTileM || row0 >= m || col0 + need > m) {
        std::printf("m=%d: tile (%d, %d, %d) off the grid\n", m, row0, col0, need);
        bad = true;
        return;
      }
      const bool transposed = col0 > row0;
      if (row0 + kTileM > m && !(col0 == row0 && !transposed)) {
        std::printf("m=%d: tile (%d, %d) has ragged rows off the diagonal\n", m, row0, col0);
        bad = true;
      }
      for (int i = row0; i < row0 + kTileM && i < m; ++i)
        for (int j = col0; j < col0 + need; ++j) {
          const int r = transposed ? j : i, c = transposed ? i : j;
          if (c > r) continue;  // the upper half of a diagonal tile is not an output
          if (++cover[static_cast<size_t>(r) * m + c] > 1) {
            std::printf("m=%d: element (%d, %d) covered twice\n", m, r, c);
            bad = true;
            return;
          }
        }
    });
    for (int r = 0; r < m && !bad; ++r)
      for (int c = 0; c <= r; ++c)
        if (cover[static_cast<size_t>(r) * m + c] != 1) {
          std::printf("m=%d: element (%d, %d) not covered\n", m, r, c);
          bad = true;
          break;
        }
    if (bad) return 1;
    if (m == 1408) tiles_1408 = count;
  }
  std::printf("ok %d\n", tiles_1408);
  return 0;
}
