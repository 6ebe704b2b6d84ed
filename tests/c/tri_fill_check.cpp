// CPU check of the triangle-clearing launches: runs the kernels' index arithmetic (tri_row_span
// and fill_span from tri_fill.cuh, the loops of zero_lower_kernel and zero_upper_kernel) over a
// launch grid of GRID blocks of 256 threads on a matrix of ones and prints the 0/1 matrix (one row
// per line). Usage: tri_fill_check PART D LD GRID
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "tri_fill.cuh"

int main(int argc, char** argv) {
  if (argc != 5) return 2;
  const int part = std::atoi(argv[1]), d = std::atoi(argv[2]);
  const long long ld = std::atoll(argv[3]);
  const int grid = std::atoi(argv[4]);
  std::vector<float> M((size_t)d * ld, 1.0f);
  const int block = 256;
  for (int b = 0; b < grid; ++b)
    for (int t = 0; t < block; ++t)
      for (long long r = b; r < d; r += grid) {
        long long lo, hi;
        gptq::tri_row_span(part, r, d, lo, hi);
        gptq::fill_span(M.data() + r * ld, lo, hi, 0.0f, t, block);
      }
  for (int r = 0; r < d; ++r) {
    for (long long c = 0; c < ld; ++c) std::putchar(M[(size_t)r * ld + c] == 0.0f ? '0' : '1');
    std::putchar('\n');
  }
  return 0;
}
