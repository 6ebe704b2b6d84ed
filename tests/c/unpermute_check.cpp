// CPU check of the codes unpermutation: runs unpermute_codes_kernel's loops (tri_row_span and
// unpermute_elem from tri_fill.cuh) over the host's launch grid.
// Usage: unpermute_check N D cs.bin perm.bin out.bin
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "tri_fill.cuh"

int main(int argc, char** argv) {
  if (argc != 6) return 2;
  const int n = std::atoi(argv[1]), d = std::atoi(argv[2]);
  std::vector<unsigned char> cs((size_t)n * d), codes((size_t)n * d, 255);
  std::vector<int> perm(d);
  FILE* f = std::fopen(argv[3], "rb");
  if (!f || std::fread(cs.data(), 1, cs.size(), f) != cs.size()) return 3;
  std::fclose(f);
  f = std::fopen(argv[4], "rb");
  if (!f || std::fread(perm.data(), 4, perm.size(), f) != perm.size()) return 3;
  std::fclose(f);
  const int block = 256, gx = (d + 1023) / 1024, gy = n < 65535 ? n : 65535;
  for (int by = 0; by < gy; ++by)
    for (int bx = 0; bx < gx; ++bx)
      for (int tx = 0; tx < block; ++tx)
        for (long long r = by; r < n; r += gy) {
          long long lo, hi;
          gptq::tri_row_span(gptq::kWholeRow, r, d, lo, hi);
          for (long long k = lo + (long long)bx * block + tx; k < hi; k += (long long)gx * block)
            gptq::unpermute_elem(cs.data(), perm.data(), codes.data(), d, r, k);
        }
  f = std::fopen(argv[5], "wb");
  if (!f || std::fwrite(codes.data(), 1, codes.size(), f) != codes.size()) return 3;
  std::fclose(f);
  return 0;
}
