// CPU check of gemv_pairs.cuh: reads N runs of BITS words, writes for each run the 32 codes as
// the tensor-core GEMV's pairs place them (by column index within the run). Exits non-zero if a
// pair is not two clean in-place fields (code << pos in each half, pos + BITS <= 10), if a
// column is covered twice, or if the two pairs of an MMA differ in class.
// Usage: gemv_pairs_check BITS N IN OUT
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "gemv_pairs.cuh"

template <int BITS>
int run(int n, const std::vector<uint32_t>& in, std::vector<uint8_t>& out) {
  using PS = gptq::PairSet<BITS>;
  for (int q = 0; q < 8; ++q)
    if (PS::pair(2 * q).cls != PS::cls(q) || PS::pair(2 * q + 1).cls != PS::cls(q)) return 10;
  for (int r = 0; r < n; ++r) {
    const uint32_t* w = in.data() + (size_t)r * BITS;
    int seen[32] = {0};
    for (int p = 0; p < 16; ++p) {
      const gptq::PairDesc d = PS::pair(p);
      const int pos = (BITS != 3 && d.cls) ? PS::POS1 : 0;
      if (pos + BITS > 10 || d.j1 < 0 || d.j1 > 31 || d.j2 < 0 || d.j2 > 31) return 11;
      const uint32_t v = gptq::pair_code<BITS>(w, p);
      const uint32_t lo = v & 0xFFFFu, hi = v >> 16;
      const uint32_t c1 = lo >> pos, c2 = hi >> pos;
      if ((c1 << pos) != lo || (c2 << pos) != hi || c1 >= (1u << BITS) || c2 >= (1u << BITS))
        return 12;
      ++seen[d.j1];
      ++seen[d.j2];
      out[(size_t)r * 32 + d.j1] = (uint8_t)c1;
      out[(size_t)r * 32 + d.j2] = (uint8_t)c2;
    }
    for (int j = 0; j < 32; ++j)
      if (seen[j] != 1) return 13;
  }
  return 0;
}

int main(int argc, char** argv) {
  if (argc != 5) return 2;
  const int bits = std::atoi(argv[1]), n = std::atoi(argv[2]);
  std::vector<uint32_t> in((size_t)n * bits);
  std::vector<uint8_t> out((size_t)n * 32);
  FILE* f = std::fopen(argv[3], "rb");
  if (!f || std::fread(in.data(), 4, in.size(), f) != in.size()) return 3;
  std::fclose(f);
  int rc = 2;
  switch (bits) {
    case 2: rc = run<2>(n, in, out); break;
    case 3: rc = run<3>(n, in, out); break;
    case 4: rc = run<4>(n, in, out); break;
    case 8: rc = run<8>(n, in, out); break;
  }
  if (rc) return rc;
  f = std::fopen(argv[4], "wb");
  if (!f || std::fwrite(out.data(), 1, out.size(), f) != out.size()) return 4;
  std::fclose(f);
  return 0;
}
