// gemv_pairs.cuh — how the tensor-core GEMV cuts a lane's run of 32 packed codes into 16 fp16
// pairs for its MMAs. Host-and-device code, so that the CPU checks run the decoding the kernel
// uses.
//
// Decoding without a subtraction. An fp16 bit pattern with a zero exponent field is the
// subnormal value mantissa * 2^-24, so a field of BITS bits masked in place at bit position pos
// of both 16-bit halves of a word (pos + BITS <= 10) is, as it stands, the fp16 pair
// (code_lo, code_hi) * 2^(pos - 24): exact, one AND per two codes (plus a shift of the word that
// serves several pairs). The MMAs of one accumulator class all use fields at the same pos, so the
// class's sum is sum(code * x) * 2^(pos - 24); the zero point enters once per chunk as
// z * sum(x).
//
// A lane's 32 columns of a row (its run: BITS words, code k at stream bits [BITS k, BITS k +
// BITS)) give 16 pairs. Pair p holds the codes (j1, j2) of the run in its low and high half;
// MMA q (one 16-wide k-step) takes pairs 2q (k slots 2t, 2t + 1) and 2q + 1 (slots 2t + 8,
// 2t + 9), and the activation pairs of the same columns: the dot product does not depend on the
// order of its terms, only A and B must agree.
//   4-bit  word i: (w & 0x000F000F) = codes (8i, 8i+4), (w >> 8) & 0x000F000F = (8i+2, 8i+6)
//          [class 0, pos 0]; masks 0x00F000F0 give (8i+1, 8i+5), (8i+3, 8i+7) [class 1, pos 4].
//   2-bit  word i: shifts 0, 2, 8, 10 with mask 0x00030003 [class 0] or 0x00300030 [class 1].
//   8-bit  word i: (w & 0x00FF00FF) = (4i, 4i+2), (w >> 8) & 0x00FF00FF = (4i+1, 4i+3).
//   3-bit  pair p: codes (2p, 2p+1), the 6 bits at stream bit 6p (joined across the two words
//          they straddle), the second code moved from bits 3-5 to bits 16-18.
#pragma once

#include <stdint.h>

#include "hd.cuh"

namespace gptq {

struct PairDesc {
  int word, shift, cls;  // value: (w[word] >> shift) & mask of the class (3-bit: see pair_code)
  int j1, j2;            // codes of the run in the low and the high half
};

template <int BITS>
struct PairSet {
  static constexpr int NCLS = (BITS == 2 || BITS == 4) ? 2 : 1;
  static constexpr int POS1 = 4;  // class 1 fields sit at bit 4 of each half (class 0: bit 0)
  // Class of MMA q (both of its pairs have it).
  static constexpr int cls(int q) {
    return BITS == 4 ? (q & 1) : (BITS == 2 ? ((q & 3) >> 1) : 0);
  }
  static constexpr PairDesc pair(int p) {
    if (BITS == 4) {
      const int i = p >> 2, k = p & 3;  // k: 0 -> (0, 4), 1 -> (2, 6), 2 -> (1, 5), 3 -> (3, 7)
      const int sh = (k & 1) ? 8 : 0, c = k >> 1;
      const int j = (k & 1) * 2 + c;
      return PairDesc{i, sh, c, 8 * i + j, 8 * i + j + 4};
    } else if (BITS == 2) {
      const int i = p >> 3, k = p & 7;  // k 0..3: class 0, codes 0, 1, 4, 5 (+ 8); 4..7: class 1
      const int c = k >> 2, r = k & 3;
      const int sh = (r & 1) * 2 + (r >> 1) * 8;
      const int j = (r & 1) + (r >> 1) * 4 + 2 * c;
      return PairDesc{i, sh, c, 16 * i + j, 16 * i + j + 8};
    } else if (BITS == 8) {
      const int i = p >> 1, k = p & 1;
      return PairDesc{i, 8 * k, 0, 4 * i + k, 4 * i + k + 2};
    } else {  // 3-bit: consecutive codes; word and shift locate stream bit 6p
      return PairDesc{(6 * p) >> 5, (6 * p) & 31, 0, 2 * p, 2 * p + 1};
    }
  }
};

// Pair p of a run held in BITS words, as the fp16 pattern of (code_j1, code_j2) * 2^(pos - 24).
template <int BITS>
GPTQ_HD uint32_t pair_code(const uint32_t* w, int p) {
  const PairDesc d = PairSet<BITS>::pair(p);
  if (BITS == 3) {
    uint32_t v = w[d.word] >> d.shift;
    if (d.shift + 6 > 32) v |= w[d.word + 1] << (32 - d.shift);
    return (v & 7u) | (((v >> 3) & 7u) << 16);
  }
  const uint32_t fm = (1u << BITS) - 1u;
  const uint32_t m0 = fm | (fm << 16);
  return (w[d.word] >> d.shift) & (d.cls ? (m0 << PairSet<BITS>::POS1) : m0);
}

}  // namespace gptq
