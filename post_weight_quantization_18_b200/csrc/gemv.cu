// gemv.cu — dequantizing matrix-vector product on the packed format (the W4A16 / W3A16 consumer
// of gptq_pack's output).
//
// "GPTQ: Mathematical Foundations ...", §Inference Execution and Modern Kernel Architectures:
// packed codes are streamed from HBM, unpacked with bit shifts and dequantized in registers,
// w_hat = (q - z) * s with the FP16 scale and zero, and multiplied with the FP16 activations,
// accumulating in higher precision (fused dequantize-and-GEMV for low-batch decoding).
//
// Y[b, r] = sum_c (code[r, c] - z[r, G(c)]) * s[r, G(c)] * X[b, c], b < batch <= 8, with
// G(c) = g_idx[c], or c / group_size when g_idx is NULL (0 for one group per row).
//
// Layout: one warp per output row. A row of qweight is one LSB-first bit stream along d_in
// (code k at stream bits [b k, b k + b)); lane l takes runs of 32 codes, i.e. exactly BITS words,
// run l, l + 32, ..., so a warp reads 128 * BITS contiguous bytes per step (16-byte loads for
// 4 and 8 bits). The 32 codes of a run come out of the BITS words with compile-time shifts (a
// 3-bit code may straddle two words) and become exact fp32 values code - z by the 2^23
// exponent trick. With contiguous groups of at least 32 columns a run lies in one group:
// Y += s * sum (q - z) x; otherwise the parameters are looked up per column. Activations are
// read 8 halves at a time; all sums are fp32, added across the warp with shuffles.
//
// Tensor-core path (2-, 4- and 8-bit codes, contiguous groups that are whole multiples of
// 128 columns or one group per row, d_in a multiple of 128): a CTA owns 16 output rows and its
// warps split d_in into 128-column chunks. Per chunk a warp issues 8 mma.sync m16n8k16 (fp16 in,
// fp32 accumulate) with A = code - z (16 rows x 16 columns) and B = X (16 columns x 8 batch
// rows, zero beyond the batch). Lane (g, t) holds rows g and g + 8 and the 32 columns
// [32 t, 32 t + 32) of the chunk, which are exactly `bits` packed words per row. Because the
// dot product sums over columns, the order in which those 32 columns enter the MMA's k slots is
// free as long as A and B use the same one: a word of 32 / bits codes gives the fp16 pairs
// (code j, code j + 16 / bits) with one mask-and-or, 0x6400 | (code << pos) being the fp16
// value 1024 + code * 2^pos, and one half2 fma with 2^-pos and -(1024 * 2^-pos + z) leaves
// code - z exactly (integers below 2^11); a shift of the word is needed only once the field
// would leave the 10-bit mantissa. The activations take the same pairing with byte permutes.
// Warps per CTA (4, 6 or 8) are the most that keep every tile resident. The 8 k-steps of a chunk
// accumulate in fp32 on the tensor core; the chunk's sum is then scaled by its group's s in
// fp32. The warps' partial sums are added in a fixed order through shared memory.
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"

namespace {

constexpr int GEMV_THREADS = 256;
constexpr int kMaxBatch = 8;

template <int BITS>
__device__ __forceinline__ void load_run(const uint32_t* __restrict__ src, uint32_t (&w)[BITS]) {
  if constexpr (BITS == 4) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(src));
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if constexpr (BITS == 8) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(src));
    const uint4 b = __ldg(reinterpret_cast<const uint4*>(src) + 1);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  } else if constexpr (BITS == 2) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(src));
    w[0] = v.x; w[1] = v.y;
  } else {
#pragma unroll
    for (int i = 0; i < BITS; ++i) w[i] = __ldg(src + i);
  }
}

// Code k (0..31) of a run held in BITS words, as an integer.
template <int BITS, int K>
__device__ __forceinline__ uint32_t code_bits(const uint32_t (&w)[BITS]) {
  constexpr int bit = K * BITS, wi = bit / 32, off = bit % 32;
  constexpr uint32_t mask = (1u << BITS) - 1u;
  uint32_t v = w[wi] >> off;
  if constexpr (off + BITS > 32) v |= w[wi + 1] << (32 - off);
  return v & mask;
}

// code - z, exact in fp32: 2^23 + code is the float with bit pattern 0x4B000000 | code, and
// zoff = 2^23 + z is exact for integer z < 2^23.
template <int BITS, int K>
__device__ __forceinline__ float code_minus_z(const uint32_t (&w)[BITS], float zoff) {
  return __uint_as_float(0x4B000000u | code_bits<BITS, K>(w)) - zoff;
}

template <int BITS, int K = 0>
__device__ __forceinline__ void codes_minus_z(const uint32_t (&w)[BITS], float zoff,
                                              float (&qz)[32]) {
  if constexpr (K < 32) {
    qz[K] = code_minus_z<BITS, K>(w, zoff);
    codes_minus_z<BITS, K + 1>(w, zoff, qz);
  }
}

// dot of 32 fp32 values with 32 fp16 activations at x (16-byte aligned).
__device__ __forceinline__ float dot32(const float (&qz)[32], const __half* __restrict__ x) {
  const uint4* xp = reinterpret_cast<const uint4*>(x);
  float dot = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 v = __ldg(xp + i);
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[j]));
      dot = fmaf(qz[8 * i + 2 * j], f.x, dot);
      dot = fmaf(qz[8 * i + 2 * j + 1], f.y, dot);
    }
  }
  return dot;
}

// One run of 32 columns starting at c0: acc[b] += sum_k w_hat[k] X[b, c0 + k].
template <int BITS, int MAXB>
__device__ __forceinline__ void run_dot(const uint32_t (&w)[BITS], int c0, bool run_groups,
                                        const __half* __restrict__ srow,
                                        const __half* __restrict__ zrow, int group_size,
                                        const int32_t* __restrict__ g_idx,
                                        const __half* __restrict__ X, long long ldx, int batch,
                                        float (&acc)[MAXB]) {
  float qz[32];
  if (run_groups) {
    const int gi = group_size <= 0 ? 0 : c0 / group_size;
    const float s = __half2float(srow[gi]);
    codes_minus_z<BITS>(w, 8388608.f + __half2float(zrow[gi]), qz);
#pragma unroll
    for (int b = 0; b < MAXB; ++b)
      if (b < batch) acc[b] = fmaf(s, dot32(qz, X + b * ldx + c0), acc[b]);
  } else {
    // Parameters per column: qz holds (code - z) * s.
    codes_minus_z<BITS>(w, 8388608.f, qz);
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const int c = c0 + k;
      const int gi = g_idx ? g_idx[c] : (group_size <= 0 ? 0 : c / group_size);
      qz[k] = (qz[k] - __half2float(zrow[gi])) * __half2float(srow[gi]);
    }
#pragma unroll
    for (int b = 0; b < MAXB; ++b)
      if (b < batch) acc[b] += dot32(qz, X + b * ldx + c0);
  }
}

// MAXB: the largest batch this instance handles (1 for decoding one token, kMaxBatch otherwise).
template <int BITS, int MAXB>
__global__ void __launch_bounds__(GEMV_THREADS)
dequant_gemv_kernel(const uint32_t* __restrict__ qweight, int n, int d, long long words_per_row,
                    const __half* __restrict__ scales, const __half* __restrict__ zeros, int G,
                    int group_size, const int32_t* __restrict__ g_idx,
                    const __half* __restrict__ X, long long ldx, int batch, float* __restrict__ Y,
                    long long ldy) {
  const int row = blockIdx.x * (GEMV_THREADS / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= n) return;
  const uint32_t* wrow = qweight + (long long)row * words_per_row;
  const __half* srow = scales + (long long)row * G;
  const __half* zrow = zeros + (long long)row * G;
  // Contiguous groups of >= 32 columns (or one group per row): a run lies inside one group.
  const bool run_groups = g_idx == nullptr && (group_size <= 0 || group_size % 32 == 0);
  float acc[MAXB];
#pragma unroll
  for (int b = 0; b < MAXB; ++b) acc[b] = 0.f;
  const int runs = d / 32;
  // Two runs per lane and step, both loads issued before either is used, so that twice the
  // bytes are in flight per warp.
  for (int r = lane; r < runs; r += 64) {
    uint32_t w0[BITS], w1[BITS];
    const bool has1 = r + 32 < runs;
    load_run<BITS>(wrow + (long long)r * BITS, w0);
    if (has1) load_run<BITS>(wrow + (long long)(r + 32) * BITS, w1);
    run_dot<BITS, MAXB>(w0, 32 * r, run_groups, srow, zrow, group_size, g_idx, X, ldx, batch, acc);
    if (has1)
      run_dot<BITS, MAXB>(w1, 32 * (r + 32), run_groups, srow, zrow, group_size, g_idx, X, ldx,
                          batch, acc);
  }
#pragma unroll
  for (int b = 0; b < MAXB; ++b) {
    float v = acc[b];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0 && b < batch) Y[b * ldy + row] = v;
  }
}

// ---------------------------------------------------------------------------------------------
// Tensor-core path
// ---------------------------------------------------------------------------------------------
constexpr int kChunk = 128;        // columns of one warp step (8 k-steps of 16)
constexpr int kMmaMaxWarps = 8;

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Packed words are read once: keep them out of L1, which holds the activations and the group
// parameters that every chunk re-reads.
template <int BITS>
__device__ __forceinline__ void load_stream(const uint32_t* __restrict__ src, uint32_t (&w)[BITS]) {
  if constexpr (BITS == 2) {
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                 : "=r"(w[0]), "=r"(w[1]) : "l"(src));
  } else {
#pragma unroll
    for (int i = 0; i < BITS; i += 4)
      asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                   : "=r"(w[i]), "=r"(w[i + 1]), "=r"(w[i + 2]), "=r"(w[i + 3])
                   : "l"(src + i));
  }
}

// Decoding a word without a shift per pair: a field of BITS bits at bit position pos of both
// 16-bit halves, or'ed into 0x6400, is the fp16 value 1024 + code * 2^pos as long as
// pos + BITS <= 10 (it stays in the mantissa). POS_PER_SHIFT fields fit; one shift of the word
// serves the next POS_PER_SHIFT pairs. fma(v, 2^-pos, -(1024 * 2^-pos + z)) is then code - z,
// exact in fp16 (a single rounding of an integer below 2^11).
template <int BITS>
struct Decode {
  static constexpr int CPW = 32 / BITS;                 // codes per word
  static constexpr int PAIRS = CPW / 2;                 // fp16 pairs per word
  static constexpr int POS_PER_SHIFT = (10 - BITS) / BITS + 1;
  static constexpr int NPOS = POS_PER_SHIFT < PAIRS ? POS_PER_SHIFT : PAIRS;
  static constexpr int shift(int j) { return BITS * POS_PER_SHIFT * (j / POS_PER_SHIFT); }
  static constexpr int pos(int j) { return BITS * (j % POS_PER_SHIFT); }
};

// Per-row constants -(1024 * 2^-pos + z) for the NPOS field positions, as fp16 pairs (exact:
// z is an integer below 2^BITS).
template <int BITS>
__device__ __forceinline__ void row_consts(__half z, __half2 (&c)[Decode<BITS>::NPOS]) {
#pragma unroll
  for (int k = 0; k < Decode<BITS>::NPOS; ++k) {
    const float off = 1024.f / (float)(1 << (BITS * k));
    c[k] = __half2half2(__hsub(__float2half_rn(-off), z));
  }
}

template <int BITS, int J>
__device__ __forceinline__ uint32_t pair_minus_z(uint32_t w,
                                                 const __half2 (&c)[Decode<BITS>::NPOS]) {
  using D = Decode<BITS>;
  constexpr int sh = D::shift(J), pos = D::pos(J);
  constexpr uint32_t m = ((1u << BITS) - 1u) << pos;
  const uint32_t v = ((w >> sh) & (m | (m << 16))) | 0x64006400u;
  const __half2 scale = __float2half2_rn(1.f / (float)(1 << pos));
  const __half2 h =
      __hfma2(*reinterpret_cast<const __half2*>(&v), scale, c[J % D::POS_PER_SHIFT]);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Word I of the lane's share of a chunk: CPW/4 k-steps. Pair 2s fills k slots 2t, 2t+1 and pair
// 2s+1 slots 2t+8, 2t+9; the activations of those columns are paired the same way.
template <int BITS, int I, int S = 0>
__device__ __forceinline__ void word_steps(uint32_t wa, uint32_t wb, const uint32_t (&xr)[16],
                                           const __half2 (&ca)[Decode<BITS>::NPOS],
                                           const __half2 (&cb)[Decode<BITS>::NPOS],
                                           float (&d0)[4], float (&d1)[4]) {
  constexpr int CPW = Decode<BITS>::CPW;
  if constexpr (S < CPW / 4) {
    const uint32_t a0 = pair_minus_z<BITS, 2 * S>(wa, ca);
    const uint32_t a1 = pair_minus_z<BITS, 2 * S>(wb, cb);
    const uint32_t a2 = pair_minus_z<BITS, 2 * S + 1>(wa, ca);
    const uint32_t a3 = pair_minus_z<BITS, 2 * S + 1>(wb, cb);
    constexpr int r = I * CPW / 2 + S;
    const uint32_t b0 = __byte_perm(xr[r], xr[r + CPW / 4], 0x5410);
    const uint32_t b1 = __byte_perm(xr[r], xr[r + CPW / 4], 0x7632);
    if constexpr (((I * (CPW / 4) + S) & 1) == 0)
      mma_16816(d0, a0, a1, a2, a3, b0, b1);
    else
      mma_16816(d1, a0, a1, a2, a3, b0, b1);
    word_steps<BITS, I, S + 1>(wa, wb, xr, ca, cb, d0, d1);
  }
}

template <int BITS, int I = 0>
__device__ __forceinline__ void chunk_words(const uint32_t (&wa)[BITS],
                                            const uint32_t (&wb)[BITS], const uint32_t (&xr)[16],
                                            const __half2 (&ca)[Decode<BITS>::NPOS],
                                            const __half2 (&cb)[Decode<BITS>::NPOS],
                                            float (&d0)[4], float (&d1)[4]) {
  if constexpr (I < BITS) {
    word_steps<BITS, I>(wa[I], wb[I], xr, ca, cb, d0, d1);
    chunk_words<BITS, I + 1>(wa, wb, xr, ca, cb, d0, d1);
  }
}

// Group parameters of rows g and g + 8.
struct GroupParams {
  __half sa, sb, za, zb;
};

// The ring holds 2 * BURST chunks of packed words per lane; BURST consecutive chunks (BURST *
// 64 contiguous bytes of a row for 4-bit codes) are requested back to back. Measured on B200 at
// 8192 x 28672, 4-bit: BURST 1 (76 registers, six warps per CTA, one wave) beats BURST 2
// (98 registers, fewer warps) and a forced 80-register BURST 2 (spills).
template <int BITS, int BURST>
__global__ void __launch_bounds__(kMmaMaxWarps * 32)
dequant_gemv_mma_kernel(const uint32_t* __restrict__ qweight, int n, int d, long long wpr,
                        const __half* __restrict__ scales, const __half* __restrict__ zeros,
                        int G, int chunks_per_group, const __half* __restrict__ X, long long ldx,
                        int batch, float* __restrict__ Y, long long ldy) {
  using D = Decode<BITS>;
  __shared__ float4 red[kMmaMaxWarps][32];
  const int nw = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int row0 = blockIdx.x * 16;
  // Rows past the end read the last row (valid memory) and are not written; batch rows past the
  // batch read the last batch row and land in accumulator columns that are not written.
  const int ra = min(row0 + g, n - 1), rb = min(row0 + g + 8, n - 1);
  const int chunks = d / kChunk;
  const int c_begin = (int)((long long)chunks * warp / nw);
  const int c_end = (int)((long long)chunks * (warp + 1) / nw);
  const int nc = c_end - c_begin;
  constexpr int CW = kChunk * BITS / 32;  // words of one row in a chunk
  const uint32_t* pa = qweight + (long long)ra * wpr + t * BITS + (long long)c_begin * CW;
  const uint32_t* pb = qweight + (long long)rb * wpr + t * BITS + (long long)c_begin * CW;
  const __half* xp =
      X + (long long)min(g, batch - 1) * ldx + 32 * t + (long long)c_begin * kChunk;
  const __half* sa = scales + (long long)ra * G;
  const __half* sb = scales + (long long)rb * G;
  const __half* za = zeros + (long long)ra * G;
  const __half* zb = zeros + (long long)rb * G;

  uint32_t wa[2][BURST][BITS], wb[2][BURST][BITS];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int k = 0; k < BURST; ++k)
      if (h * BURST + k < nc) {
        load_stream<BITS>(pa + (h * BURST + k) * CW, wa[h][k]);
        load_stream<BITS>(pb + (h * BURST + k) * CW, wb[h][k]);
      }

  // Group bookkeeping without a division per chunk; the next group's parameters are fetched
  // when a group starts. (A warp with no chunks reads group 0, which exists.)
  int gi = c_begin / chunks_per_group;
  if (gi >= G) gi = G - 1;
  int g_next = (gi + 1) * chunks_per_group;  // first chunk of the next group
  GroupParams cur{sa[gi], sb[gi], za[gi], zb[gi]};
  GroupParams nxt = cur;
  if (gi + 1 < G) nxt = GroupParams{sa[gi + 1], sb[gi + 1], za[gi + 1], zb[gi + 1]};
  __half2 ca[D::NPOS], cb[D::NPOS];
  row_consts<BITS>(cur.za, ca);
  row_consts<BITS>(cur.zb, cb);
  float s_a = __half2float(cur.sa), s_b = __half2float(cur.sb);

  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int base = 0; base < nc; base += 2 * BURST) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int k = 0; k < BURST; ++k) {
        const int ci = base + h * BURST + k;
        if (ci < nc) {
          if (c_begin + ci == g_next) {
            ++gi;
            g_next += chunks_per_group;
            cur = nxt;
            if (gi + 1 < G) nxt = GroupParams{sa[gi + 1], sb[gi + 1], za[gi + 1], zb[gi + 1]};
            row_consts<BITS>(cur.za, ca);
            row_consts<BITS>(cur.zb, cb);
            s_a = __half2float(cur.sa);
            s_b = __half2float(cur.sb);
          }
          uint32_t xr[16];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(xp + ci * kChunk) + i);
            xr[4 * i] = v.x; xr[4 * i + 1] = v.y; xr[4 * i + 2] = v.z; xr[4 * i + 3] = v.w;
          }
          float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
          chunk_words<BITS>(wa[h][k], wb[h][k], xr, ca, cb, d0, d1);
          acc[0] = fmaf(s_a, d0[0] + d1[0], acc[0]);
          acc[1] = fmaf(s_a, d0[1] + d1[1], acc[1]);
          acc[2] = fmaf(s_b, d0[2] + d1[2], acc[2]);
          acc[3] = fmaf(s_b, d0[3] + d1[3], acc[3]);
        }
      }
#pragma unroll
      for (int k = 0; k < BURST; ++k) {
        const int cn = base + (h + 2) * BURST + k;
        if (cn < nc) {
          load_stream<BITS>(pa + cn * CW, wa[h][k]);
          load_stream<BITS>(pb + cn * CW, wb[h][k]);
        }
      }
    }
  }
  red[warp][lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
  __syncthreads();
  if (warp != 0) return;
  for (int w = 1; w < nw; ++w) {
    const float4 v = red[w][lane];
    acc[0] += v.x; acc[1] += v.y; acc[2] += v.z; acc[3] += v.w;
  }
  // Accumulator layout: acc[e] is (row g, batch 2t + e), acc[2 + e] is (row g + 8, batch 2t + e).
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int b = 2 * t + e;
    if (b >= batch) continue;
    if (row0 + g < n) Y[(long long)b * ldy + row0 + g] = acc[e];
    if (row0 + g + 8 < n) Y[(long long)b * ldy + row0 + g + 8] = acc[2 + e];
  }
}

}  // namespace

namespace gptq_host {

namespace {

// Warps per CTA for the tensor-core kernel: the most of 8, 6 or 4 that still lets every 16-row
// tile be resident at once (one wave); 4 when no choice fits.
template <class K>
int mma_launch(K kernel, int tiles, const uint32_t* qweight, int n, int d, long long wpr,
               const __half* s, const __half* z, int G, int cpg, const __half* x, long long ldx,
               int batch, float* y, long long ldy, cudaStream_t stream) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return GPTQ_ERR_CUDA;
  int nw = 4;
  for (int cand : {8, 6}) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, cand * 32, 0) !=
        cudaSuccess)
      return GPTQ_ERR_CUDA;
    if ((long long)per_sm * sms >= tiles) {
      nw = cand;
      break;
    }
  }
  kernel<<<tiles, nw * 32, 0, stream>>>(qweight, n, d, wpr, s, z, G, cpg, x, ldx, batch, y, ldy);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

}  // namespace

int dequant_gemv(const uint32_t* qweight, int n, int d, int bits, const uint16_t* scales_f16,
                 const uint16_t* zeros_f16, int n_groups, int group_size, const int32_t* g_idx,
                 const uint16_t* x_f16, int batch, long long ldx, float* y, long long ldy,
                 cudaStream_t stream) {
  const long long wpr = (long long)d * bits / 32;
  const dim3 grid((n + GEMV_THREADS / 32 - 1) / (GEMV_THREADS / 32));
  const __half* s = reinterpret_cast<const __half*>(scales_f16);
  const __half* z = reinterpret_cast<const __half*>(zeros_f16);
  const __half* x = reinterpret_cast<const __half*>(x_f16);
#define GEMV_LAUNCH(B, M)                                                                      \
  dequant_gemv_kernel<B, M><<<grid, GEMV_THREADS, 0, stream>>>(qweight, n, d, wpr, s, z, n_groups, \
                                                               group_size, g_idx, x, ldx, batch,   \
                                                               y, ldy)
  const bool run_groups = g_idx == nullptr && (n_groups == 1 || group_size % kChunk == 0);
  if (run_groups && d % kChunk == 0 && (bits == 2 || bits == 4 || bits == 8)) {
    const int tiles = (n + 15) / 16;
    const int cpg = n_groups == 1 ? d / kChunk : group_size / kChunk;
    switch (bits) {
      case 2:
        return mma_launch(dequant_gemv_mma_kernel<2, 2>, tiles, qweight, n, d, wpr, s, z,
                          n_groups, cpg, x, ldx, batch, y, ldy, stream);
      case 4:
        return mma_launch(dequant_gemv_mma_kernel<4, 1>, tiles, qweight, n, d, wpr, s, z,
                          n_groups, cpg, x, ldx, batch, y, ldy, stream);
      default:
        return mma_launch(dequant_gemv_mma_kernel<8, 1>, tiles, qweight, n, d, wpr, s, z,
                          n_groups, cpg, x, ldx, batch, y, ldy, stream);
    }
  }
  const bool one = batch == 1;
  switch (bits) {
    case 2: if (one) GEMV_LAUNCH(2, 1); else GEMV_LAUNCH(2, kMaxBatch); break;
    case 3: if (one) GEMV_LAUNCH(3, 1); else GEMV_LAUNCH(3, kMaxBatch); break;
    case 4: if (one) GEMV_LAUNCH(4, 1); else GEMV_LAUNCH(4, kMaxBatch); break;
    case 8: if (one) GEMV_LAUNCH(8, 1); else GEMV_LAUNCH(8, kMaxBatch); break;
    default: return GPTQ_ERR_INVALID_ARG;
  }
#undef GEMV_LAUNCH
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

}  // namespace gptq_host
