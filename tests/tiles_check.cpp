// Host check of the tile enumeration the Newton-Schulz product kernels and the
// planner share (dm_tiles.cuh).  For symmetric products the enumerated tiles
// must be exactly the tiles that meet the upper triangle, each once; for the
// other products every tile once, in the documented order.  Prints one line
// per failure and exits non-zero if there is any.
#include <cstdio>
#include <set>
#include <utility>

#include "dm_tiles.cuh"

static int check(int M, int N, int bm, int bn, int flags) {
  dm::GemmMat g{};
  g.M = M;
  g.N = N;
  g.flags = flags;
  g.tiles_m = (M + bm - 1) / bm;
  g.tiles_n = (N + bn - 1) / bn;
  const int cnt = dm::gemm_tile_count(g, bm, bn);
  std::set<std::pair<int, int>> seen;
  int bad = 0;
  for (int lt = 0; lt < cnt; ++lt) {
    int tm = -1, tn = -1;
    dm::gemm_tile_coord(g, lt, bm, bn, tm, tn);
    if (tm < 0 || tm >= g.tiles_m || tn < 0 || tn >= g.tiles_n || !seen.insert({tm, tn}).second) {
      std::printf("M %d N %d bm %d bn %d flags %d: index %d -> bad or repeated tile (%d, %d)\n", M, N,
                  bm, bn, flags, lt, tm, tn);
      ++bad;
    }
    if (!(flags & dm::GF_SYM)) {
      const int want_tm = (flags & dm::GF_N_FAST) ? lt / g.tiles_n : lt % g.tiles_m;
      const int want_tn = (flags & dm::GF_N_FAST) ? lt % g.tiles_n : lt / g.tiles_m;
      if (tm != want_tm || tn != want_tn) {
        std::printf("M %d N %d flags %d: index %d -> (%d, %d), order (%d, %d)\n", M, N, flags, lt,
                    tm, tn, want_tm, want_tn);
        ++bad;
      }
    }
  }
  for (int tm = 0; tm < g.tiles_m; ++tm)
    for (int tn = 0; tn < g.tiles_n; ++tn) {
      // the tile holds an element (r, c) with c >= r
      const bool meets = (tn * bn + bn - 1) >= tm * bm;
      const bool want = (flags & dm::GF_SYM) ? meets : true;
      if (want != (seen.count({tm, tn}) == 1)) {
        std::printf("M %d N %d bm %d bn %d flags %d: tile (%d, %d) %s\n", M, N, bm, bn, flags, tm, tn,
                    want ? "missing" : "enumerated but outside the upper triangle");
        ++bad;
      }
    }
  return bad;
}

int main() {
  const int tiles[][2] = {{128, 256}, {256, 256}, {128, 128}};
  const int sizes[] = {1, 7, 64, 127, 128, 129, 255, 256, 257, 384, 500, 768, 1000, 1024, 1100, 3072, 4096};
  int bad = 0, runs = 0;
  for (const auto& t : tiles)
    for (int m : sizes) {
      bad += check(m, m, t[0], t[1], dm::GF_SYM);
      ++runs;
      for (int n : sizes) {
        bad += check(m, n, t[0], t[1], dm::GF_N_FAST);
        bad += check(m, n, t[0], t[1], 0);
        runs += 2;
      }
    }
  std::printf("%d enumerations checked, %d failures\n", runs, bad);
  return bad == 0 ? 0 : 1;
}
