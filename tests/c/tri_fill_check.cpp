// CPU check of the triangle-clearing launches: runs the kernels' index arithmetic (tri_row_span
// from tri_fill.cuh, the loops of zero_lower_kernel) over the host's launch grid on a matrix of
// ones and prints the 0/1 matrix (one row per line). Usage: tri_fill_check PART D LD
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "tri_fill.cuh"

int main(int argc, char** argv) {
  if (argc != 4) return 2;
  const int part = std::atoi(argv[1]), d = std::atoi(argv[2]);
  const long long ld = std::atoll(argv[3]);
  std::vector<float> M((size_t)d * ld, 1.0f);
  const int block = 256, gx = (d + 1023) / 1024, gy = d < 65535 ? d : 65535;
  for (int by = 0; by < gy; ++by)
    for (int bx = 0; bx < gx; ++bx)
      for (int tx = 0; tx < block; ++tx)
        for (long long r = by; r < d; r += gy) {
          long long lo, hi;
          gptq::tri_row_span(part, r, d, lo, hi);
          float* row = M.data() + r * ld;
          for (long long c = lo + (long long)bx * block + tx; c < hi; c += (long long)gx * block)
            row[c] = 0.0f;
        }
  for (int r = 0; r < d; ++r) {
    for (long long c = 0; c < ld; ++c) std::putchar(M[(size_t)r * ld + c] == 0.0f ? '0' : '1');
    std::putchar('\n');
  }
  return 0;
}
