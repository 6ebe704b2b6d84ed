// tri_fill.cuh — which elements of a row-major square matrix a triangle-clearing launch
// writes. Rows go to the grid's y dimension (grid-stride), and the threads of the x dimension
// stride along the row's span. No per-element division: the row is known and the span is
// contiguous. Host-and-device code, so that the kernels' index arithmetic is also checked on
// the CPU.
#pragma once

#include "hd.cuh"

namespace gptq {

enum TriPart { kStrictLower = 0, kUpperWithDiag = 1, kWholeRow = 2 };

// Columns [lo, hi) of row r that belong to the part.
GPTQ_HD void tri_row_span(int part, long long r, int d, long long& lo, long long& hi) {
  if (part == kStrictLower) {
    lo = 0;
    hi = r < d ? r : d;
  } else if (part == kUpperWithDiag) {
    lo = r;
    hi = d;
  } else {
    lo = 0;
    hi = d;
  }
}

// Codes back in the original column order: codes[r][perm[k]] = cs[r][k] (rows of d codes).
GPTQ_HD void unpermute_elem(const unsigned char* cs, const int* perm, unsigned char* codes, int d,
                            long long r, long long k) {
  codes[r * d + perm[k]] = cs[r * d + k];
}

// Element (a, b), b >= a, of the permuted Hessian's upper triangle: Hp[a][b] = H[pi a][pi b],
// read from H's upper triangle (H symmetric, only i <= j stored). pa = perm[a].
GPTQ_HD void permute_sym_elem(const float* H, float* Hp, const int* perm, int d, long long a,
                              int pa, long long b) {
  const int j = perm[b];
  const long long lo = pa < j ? pa : j, hi = pa < j ? j : pa;
  Hp[a * d + b] = H[lo * d + hi];
}

}  // namespace gptq
