// Tile enumeration shared by the Newton-Schulz product kernels and the host
// planner.  Symmetric products (X X^T and A A, both symmetric) visit only the
// output tiles that meet the upper triangle; every element (r, c) with c >= r
// is then written by exactly one tile, and its mirror (c, r) by the same tile.
#pragma once

#include "dm_internal.h"

namespace dm {

// First column tile of row tile tm that meets the upper triangle:
// the smallest tn with bn * (tn + 1) > bm * tm.
__host__ __device__ __forceinline__ int sym_first_tn(int tm, int bm, int bn) {
  return (bm * tm) / bn;
}

__host__ __device__ __forceinline__ int gemm_tile_count(const GemmMat& g, int bm, int bn) {
  if (!(g.flags & GF_SYM)) return g.tiles_m * g.tiles_n;
  int n = 0;
  for (int tm = 0; tm < g.tiles_m; ++tm) {
    const int f = sym_first_tn(tm, bm, bn);
    if (f < g.tiles_n) n += g.tiles_n - f;
  }
  return n;
}

// Local tile index -> (tm, tn).
__host__ __device__ __forceinline__ void gemm_tile_coord(const GemmMat& g, int lt, int bm, int bn,
                                                         int& tm, int& tn) {
  if (g.flags & GF_SYM) {
    int rem = lt;
    for (tm = 0; tm < g.tiles_m; ++tm) {
      const int f = sym_first_tn(tm, bm, bn);
      const int cnt = f < g.tiles_n ? g.tiles_n - f : 0;
      if (rem < cnt) {
        tn = f + rem;
        return;
      }
      rem -= cnt;
    }
    tm = tn = 0;  // unreachable for a valid index
  } else if (g.flags & GF_N_FAST) {
    tm = lt / g.tiles_n;
    tn = lt % g.tiles_n;
  } else {
    tn = lt / g.tiles_m;
    tm = lt % g.tiles_m;
  }
}

}  // namespace dm
