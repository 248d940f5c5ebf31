// Host-side check of the GEMMs' raster order (test code): for many token-
// and weight-tile counts, tile_coords (csrc/ptx.cuh) with the group size
// raster_group (csrc/internal.cuh) picks visits every (token tile, weight
// tile) exactly once; every group's activation rows fit the budget; groups
// differ in size by at most one tile; inside a group the token tiles of one
// weight tile are consecutive. Prints "ok <cases>" or the first failure.
#include <cstdio>
#include <vector>

#include "internal.cuh"
#include "ptx.cuh"

using namespace fp8blk;

static int check(int mtiles, int ntn, long long bytes_per_mtile, long long budget) {
  const int gm = raster_group(mtiles, bytes_per_mtile, budget);
  if (gm < 1 || gm > mtiles) return 1;
  if (mtiles > 1 && static_cast<long long>(gm) * bytes_per_mtile > budget && gm > 1) return 2;
  const int groups = (mtiles + gm - 1) / gm;
  const int last = mtiles - (groups - 1) * gm;
  if (last < 1 || gm - last > groups) return 3;  // near-equal: the last group is not tiny
  std::vector<int> seen(static_cast<size_t>(mtiles) * ntn, 0);
  int prev_mt = -1, prev_nt = -1;
  for (int t = 0; t < mtiles * ntn; ++t) {
    int mt, nt;
    tile_coords(t, mtiles, ntn, gm, mt, nt);
    if (mt < 0 || mt >= mtiles || nt < 0 || nt >= ntn) return 4;
    if (seen[static_cast<size_t>(mt) * ntn + nt]++) return 5;
    if (t > 0 && nt == prev_nt && mt != prev_mt + 1) return 6;  // consecutive token tiles
    if (t > 0 && mt / gm == prev_mt / gm && nt < prev_nt) return 7;  // a group sweeps forward
    prev_mt = mt;
    prev_nt = nt;
  }
  return 0;
}

int main() {
  int cases = 0;
  const long long budgets[2] = {kRasterBytesW8A8, kRasterBytesW8A16};
  const long long per_mtile[4] = {128LL * 5120, 256LL * 5120 * 2, 128LL * 3000, 256LL * 3000 * 2};
  for (long long budget : budgets)
    for (long long b : per_mtile)
      for (int mtiles = 1; mtiles <= 200; mtiles += (mtiles < 40 ? 1 : 7))
        for (int ntn : {1, 3, 20, 40, 100, 200}) {
          const int r = check(mtiles, ntn, b, budget);
          ++cases;
          if (r) {
            printf("fail %d: mtiles %d ntiles %d bytes %lld budget %lld\n", r, mtiles, ntn, b, budget);
            return 1;
          }
        }
  printf("ok %d\n", cases);
  return 0;
}
