// CPU check of the pack fast path: runs the kernel's per-chunk code (pack_chunk_ptrs and
// pack32 from pack32.cuh, the functions pack_vec_kernel calls) over every chunk of a codes
// matrix, with the two 16-byte loads and the word stores done as byte copies.
// Usage: pack32_check BITS N D codes.bin words.bin   (codes: N*D bytes; words: N*D*BITS/32 u32)
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <vector>

#include "pack32.cuh"

template <int BITS>
static void run(const std::vector<uint8_t>& codes, int n, int d, std::vector<uint32_t>& words) {
  const long long items = (long long)n * (d / 32);
  for (long long item = 0; item < items; ++item) {
    const uint8_t* src;
    uint32_t* out;
    gptq::pack_chunk_ptrs<BITS>(codes.data(), words.data(), d, item, src, out);
    uint32_t c[8];
    std::memcpy(c, src, 32);  // little-endian, as the 16-byte loads on the GPU
    uint32_t w[BITS];
    gptq::pack32<BITS>(c, w);
    std::memcpy(out, w, sizeof w);
  }
}

int main(int argc, char** argv) {
  if (argc != 6) return 2;
  const int bits = std::atoi(argv[1]), n = std::atoi(argv[2]), d = std::atoi(argv[3]);
  if (d % 32 != 0) return 2;
  std::vector<uint8_t> codes((size_t)n * d);
  FILE* f = std::fopen(argv[4], "rb");
  if (!f || std::fread(codes.data(), 1, codes.size(), f) != codes.size()) return 3;
  std::fclose(f);
  std::vector<uint32_t> words((size_t)n * d * bits / 32);
  switch (bits) {
    case 2: run<2>(codes, n, d, words); break;
    case 3: run<3>(codes, n, d, words); break;
    case 4: run<4>(codes, n, d, words); break;
    case 8: run<8>(codes, n, d, words); break;
    default: return 2;
  }
  f = std::fopen(argv[5], "wb");
  if (!f || std::fwrite(words.data(), 4, words.size(), f) != words.size()) return 3;
  std::fclose(f);
  return 0;
}
