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

}  // namespace

namespace gptq_host {

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
