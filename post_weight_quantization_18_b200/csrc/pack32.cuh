// pack32.cuh — 32 codes -> BITS packed words, the bit-stream layout of the pack format.
//
// "GPTQ: Mathematical Foundations ...", §Inference Execution and Modern Kernel Architectures
// (eight 4-bit weights per int32): a row is one LSB-first bit stream along d_in, code k at
// stream bits [BITS*k, BITS*k + BITS); 32 codes fill exactly BITS words. Host-and-device code,
// so that the same function is also checked on the CPU.
#pragma once

#include <stdint.h>

#include "hd.cuh"

namespace gptq {

// c[i] holds codes 4i .. 4i+3 as its bytes 0 .. 3 (the order 32 uint8 codes have in memory);
// only the low BITS bits of each byte are packed.
template <int BITS>
GPTQ_HD void pack32(const uint32_t (&c)[8], uint32_t (&w)[BITS]) {
  constexpr uint32_t mask = (1u << BITS) - 1u;
GPTQ_UNROLL
  for (int i = 0; i < BITS; ++i) w[i] = 0u;
GPTQ_UNROLL
  for (int k = 0; k < 32; ++k) {
    const uint32_t code = (c[k >> 2] >> (8 * (k & 3))) & mask;
    const int bit = k * BITS, wi = bit >> 5, off = bit & 31;
    w[wi] |= code << off;
    if (off + BITS > 32) w[wi + 1] |= code >> (32 - off);
  }
}

// Source and destination of chunk `item` (row item / chunks, chunk item % chunks) of a codes
// matrix [n, d] with d a multiple of 32, packed into rows of d * BITS / 32 words.
template <int BITS>
GPTQ_HD void pack_chunk_ptrs(const uint8_t* codes, uint32_t* qweight, int d, long long item,
                             const uint8_t*& src, uint32_t*& out) {
  const int chunks = d / 32;
  const long long r = item / chunks;
  const long long ch = item % chunks;
  src = codes + r * d + ch * 32;
  out = qweight + r * ((long long)d * BITS / 32) + ch * BITS;
}

}  // namespace gptq
