// CPU check of the sweep's W gather: runs the kernel's per-thread code (gather4_cols and
// gather4_row from gather4.cuh, the functions gather_w_kernel calls) over the launch grid that
// the host uses (x: d/4 columns in blocks of 256 threads, y: min(n, 65535) rows, grid-stride).
// Usage: gather4_check DTYPE(f32|bf16) N D LDW w.bin perm.bin dead.bin out.bin
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <vector>

#include "gather4.cuh"

template <typename T>
static void run(const std::vector<T>& W, long long ldw, int n, int d,
                const std::vector<int32_t>& perm, const std::vector<uint8_t>& dead,
                std::vector<float>& out) {
  const int gx = (d / 4 + 255) / 256, gy = n < 65535 ? n : 65535;
  for (int bx = 0; bx < gx; ++bx)
    for (int by = 0; by < gy; ++by)
      for (int tx = 0; tx < 256; ++tx) {
        const int k0 = 4 * (bx * 256 + tx);
        if (k0 >= d) continue;
        int32_t src[4];
        bool live[4];
        gptq::gather4_cols(perm.data(), dead.data(), k0, src, live);
        for (long long r = by; r < n; r += gy) {
          float v[4];
          gptq::gather4_row<T>(W.data(), ldw, r, src, live, v);
          std::memcpy(&out[(size_t)r * d + k0], v, sizeof v);
        }
      }
}

template <typename V>
static bool read_all(const char* path, std::vector<V>& v) {
  FILE* f = std::fopen(path, "rb");
  if (!f) return false;
  const size_t got = std::fread(v.data(), sizeof(V), v.size(), f);
  std::fclose(f);
  return got == v.size();
}

int main(int argc, char** argv) {
  if (argc != 9) return 2;
  const bool bf16 = std::strcmp(argv[1], "bf16") == 0;
  const int n = std::atoi(argv[2]), d = std::atoi(argv[3]);
  const long long ldw = std::atoll(argv[4]);
  if (d % 128 != 0) return 2;
  std::vector<int32_t> perm(d);
  std::vector<uint8_t> dead(d);
  if (!read_all(argv[6], perm) || !read_all(argv[7], dead)) return 3;
  std::vector<float> out((size_t)n * d, -1.0f);
  if (bf16) {
    std::vector<uint16_t> W((size_t)n * ldw);
    if (!read_all(argv[5], W)) return 3;
    run<uint16_t>(W, ldw, n, d, perm, dead, out);
  } else {
    std::vector<float> W((size_t)n * ldw);
    if (!read_all(argv[5], W)) return 3;
    run<float>(W, ldw, n, d, perm, dead, out);
  }
  FILE* f = std::fopen(argv[8], "wb");
  if (!f || std::fwrite(out.data(), 4, out.size(), f) != out.size()) return 3;
  std::fclose(f);
  return 0;
}
