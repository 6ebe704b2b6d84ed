// tri_fill.cuh — which elements of a row-major square matrix a triangle launch touches. The
// fills (zeroing a triangle) give each block whole rows (grid-stride over rows) and stride its
// threads along the row's span with 16-byte stores; the element-wise copies put rows on the
// grid's y dimension and stride the x dimension's threads along the span. No per-element
// division: the row is known and the span is contiguous. Host-and-device code, so that the
// kernels' index arithmetic is also checked on the CPU.
#pragma once

#include <stdint.h>

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

// Thread t of nt writes v into elements [lo, hi) of the row at p: a scalar head up to the first
// 16-byte boundary, 16-byte stores for the body, a scalar tail. (The host build, used by the
// CPU checks, writes the body's four values one by one at the same indices.)
GPTQ_HD void fill_span(float* p, long long lo, long long hi, float v, int t, int nt) {
  const long long mis = (long long)((reinterpret_cast<uintptr_t>(p + lo) >> 2) & 3);
  long long body0 = lo + ((4 - mis) & 3);
  if (body0 > hi) body0 = hi;
  for (long long c = lo + t; c < body0; c += nt) p[c] = v;
  const long long quads = (hi - body0) / 4;
  for (long long k = t; k < quads; k += nt) {
#if defined(__CUDA_ARCH__)
    reinterpret_cast<float4*>(p + body0)[k] = make_float4(v, v, v, v);
#else
    for (int e = 0; e < 4; ++e) p[body0 + 4 * k + e] = v;
#endif
  }
  for (long long c = body0 + 4 * quads + t; c < hi; c += nt) p[c] = v;
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
