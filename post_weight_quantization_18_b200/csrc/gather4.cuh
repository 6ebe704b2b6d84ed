// gather4.cuh — the working copy of W in sweep order: Wwork[r][k] = dead[k] ? 0 : W[r][perm[k]]
// as fp32 (bf16 widened exactly), four consecutive columns k0 .. k0+3 per thread. Host-and-
// device code, so that the kernel's per-thread work is also checked on the CPU.
#pragma once

#include <stdint.h>
#include <string.h>

#include "hd.cuh"

namespace gptq {

GPTQ_HD float widen(float x) { return x; }

// bf16 bit pattern -> fp32: the 16 bits are the top half of the fp32 pattern (exact).
GPTQ_HD float widen(uint16_t b) {
  const uint32_t u = (uint32_t)b << 16;
#if defined(__CUDA_ARCH__)
  return __uint_as_float(u);
#else
  float f;
  memcpy(&f, &u, 4);
  return f;
#endif
}

// Source columns of k0 .. k0+3 and whether each is live (not dead).
GPTQ_HD void gather4_cols(const int32_t* perm, const uint8_t* dead, int k0, int32_t (&src)[4],
                          bool (&live)[4]) {
GPTQ_UNROLL
  for (int j = 0; j < 4; ++j) {
    src[j] = perm[k0 + j];
    live[j] = dead[k0 + j] == 0;
  }
}

template <typename T>  // float, or uint16_t holding bf16 bit patterns
GPTQ_HD void gather4_row(const T* W, long long ldw, long long r, const int32_t (&src)[4],
                         const bool (&live)[4], float (&v)[4]) {
  const T* wr = W + r * ldw;
GPTQ_UNROLL
  for (int j = 0; j < 4; ++j) v[j] = live[j] ? widen(wr[src[j]]) : 0.0f;
}

}  // namespace gptq
