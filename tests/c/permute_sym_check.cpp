// CPU check of the act-order permutation of H: runs permute_sym_kernel's loops (tri_row_span
// and permute_sym_elem from tri_fill.cuh) over the host's launch grid.
// Usage: permute_sym_check D h.bin perm.bin out.bin   (h: D*D fp32, upper triangle valid)
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "tri_fill.cuh"

int main(int argc, char** argv) {
  if (argc != 5) return 2;
  const int d = std::atoi(argv[1]);
  std::vector<float> H((size_t)d * d), Hp((size_t)d * d, -1.0f);
  std::vector<int> perm(d);
  FILE* f = std::fopen(argv[2], "rb");
  if (!f || std::fread(H.data(), 4, H.size(), f) != H.size()) return 3;
  std::fclose(f);
  f = std::fopen(argv[3], "rb");
  if (!f || std::fread(perm.data(), 4, perm.size(), f) != perm.size()) return 3;
  std::fclose(f);
  const int block = 256, gx = (d + 1023) / 1024, gy = d < 65535 ? d : 65535;
  for (int by = 0; by < gy; ++by)
    for (int bx = 0; bx < gx; ++bx)
      for (int tx = 0; tx < block; ++tx)
        for (long long a = by; a < d; a += gy) {
          long long lo, hi;
          gptq::tri_row_span(gptq::kUpperWithDiag, a, d, lo, hi);
          const int pa = perm[a];
          for (long long b = lo + (long long)bx * block + tx; b < hi; b += (long long)gx * block)
            gptq::permute_sym_elem(H.data(), Hp.data(), perm.data(), d, a, pa, b);
        }
  f = std::fopen(argv[4], "wb");
  if (!f || std::fwrite(Hp.data(), 4, Hp.size(), f) != Hp.size()) return 3;
  std::fclose(f);
  return 0;
}
