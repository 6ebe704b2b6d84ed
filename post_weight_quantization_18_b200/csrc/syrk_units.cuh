// syrk_units.cuh — the work units of the Hessian SYRK and their order. Host-and-device code, so
// that the CPU checks under tests/c run the same mapping the kernel uses.
//
// A unit is (tile, token range): tiles (ib, jb) with ib <= jb on an n_tb x n_tb grid of
// 256 x 256 output tiles, times n_split token ranges. The tiles are cut into groups of
// grp x grp tiles (diagonal groups keep their upper half), taken column of groups by column of
// groups; inside a group the units run range by range, so the CTAs running together work on
// one group in one token range and read only its 2 grp panels of X.
#pragma once

#include "hd.cuh"

namespace gptq {

// Number of units: n_tb (n_tb + 1) / 2 tiles times n_split ranges.
GPTQ_HD long long syrk_unit_count(int n_tb, int n_split) {
  return (long long)n_tb * (n_tb + 1) / 2 * n_split;
}

// Unit u (0 <= u < syrk_unit_count) -> tile (ib, jb) and token range `split`.
GPTQ_HD void syrk_unit_coords(long long u, int n_tb, int grp, int n_split, int& ib, int& jb,
                              int& split) {
  const int ng = (n_tb + grp - 1) / grp;
  for (int gj = 0; gj < ng; ++gj) {
    const int j0 = gj * grp, w = (n_tb - j0) < grp ? (n_tb - j0) : grp;
    for (int gi = 0; gi <= gj; ++gi) {
      const int i0 = gi * grp, h = (n_tb - i0) < grp ? (n_tb - i0) : grp;
      const int tiles = (gi < gj) ? h * w : h * (h + 1) / 2;
      const long long units = (long long)tiles * n_split;
      if (u >= units) {
        u -= units;
        continue;
      }
      split = (int)(u / tiles);
      int k = (int)(u % tiles);
      if (gi < gj) {
        ib = i0 + k / w;
        jb = j0 + k % w;
      } else {  // upper half of a diagonal group: column jj holds rows 0..jj
        int jj = 0;
        while (k > jj) {
          k -= jj + 1;
          ++jj;
        }
        ib = i0 + k;
        jb = j0 + jj;
      }
      return;
    }
  }
  ib = jb = split = 0;  // unreachable for u < syrk_unit_count
}

}  // namespace gptq
