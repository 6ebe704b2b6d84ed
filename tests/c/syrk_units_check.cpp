// CPU check of the SYRK's unit order (syrk_units.cuh, the mapping the kernel calls): prints one
// line "ib jb split" per unit u = 0 .. count-1. Usage: syrk_units_check N_TB GRP N_SPLIT
#include <cstdio>
#include <cstdlib>

#include "syrk_units.cuh"

int main(int argc, char** argv) {
  if (argc != 4) return 2;
  const int n_tb = std::atoi(argv[1]), grp = std::atoi(argv[2]), n_split = std::atoi(argv[3]);
  const long long n = gptq::syrk_unit_count(n_tb, n_split);
  for (long long u = 0; u < n; ++u) {
    int ib, jb, split;
    gptq::syrk_unit_coords(u, n_tb, grp, n_split, ib, jb, split);
    std::printf("%d %d %d\n", ib, jb, split);
  }
  return 0;
}
