// quant_pack.cu — round-to-nearest baseline and the packed storage format.
//
// RTN ("GPTQ: Mathematical Foundations ...", §Comparison: RTN; "INT4 and GPTQ Quantization",
// §Uniform INT4 Quantization and §Group Quantization): (s, z) from the original weights of each
// group of g consecutive weights of a row (or of the whole row), q = clamp(rne(w/s) + z, 0,
// 2^b - 1). fp32 with IEEE division and round-half-to-even, so the result is bit-exact.
//
// Pack ("GPTQ: Mathematical Foundations ...", §Inference Execution and Modern Kernel
// Architectures: eight 4-bit weights per int32; "INT4 and GPTQ Quantization", §Group
// Quantization: scale and zero in FP16): each row is an LSB-first bit stream, code k at bits
// [b*k, b*k + b); word w holds stream bits [32w, 32w + 32). One thread packs 32 codes, which
// fill exactly b words (pack32.cuh); rows of whole chunks take vector loads and stores.
#include <float.h>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"
#include "pack32.cuh"

namespace {

template <typename T>
__device__ __forceinline__ float ld_w(const T* p) {
  if constexpr (sizeof(T) == 2)
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p));
  else
    return *p;
}

// One warp per (row, group).
template <typename T>
__global__ void rtn_kernel(const T* __restrict__ W, long long ldw, int n, int d, int bits, int g,
                           int sym, uint8_t* __restrict__ codes, float* __restrict__ scales,
                           float* __restrict__ zeros) {
  const int G = d / g;
  const long long item = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (item >= (long long)n * G) return;
  const int r = (int)(item / G), gi = (int)(item % G);
  const T* wr = W + (long long)r * ldw + (long long)gi * g;
  float mn = FLT_MAX, mx = -FLT_MAX, am = 0.f;
  for (int k = lane; k < g; k += 32) {
    const float v = ld_w(wr + k);
    mn = fminf(mn, v);
    mx = fmaxf(mx, v);
    am = fmaxf(am, fabsf(v));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
  }
  const float maxq = (float)((1 << bits) - 1);
  float s, z;
  if (sym) {
    s = __fdiv_rn(am, (float)((1 << (bits - 1)) - 1));
    if (s == 0.f) s = 1.f;
    z = (float)(1 << (bits - 1));
  } else {
    s = __fdiv_rn(mx - mn, maxq);
    if (s == 0.f) s = 1.f;
    z = fminf(fmaxf(rintf(__fdiv_rn(-mn, s)), 0.f), maxq);
  }
  if (lane == 0) {
    scales[(long long)r * G + gi] = s;
    zeros[(long long)r * G + gi] = z;
  }
  uint8_t* cr = codes + (long long)r * d + (long long)gi * g;
  for (int k = lane; k < g; k += 32) {
    const float q = fminf(fmaxf(rintf(__fdiv_rn(ld_w(wr + k), s)) + z, 0.f), maxq);
    cr[k] = (uint8_t)q;
  }
}

// One thread per (row, chunk of 32 codes) -> `bits` words (fewer at the row's tail).
__global__ void pack_kernel(const uint8_t* __restrict__ codes, int n, int d, int bits,
                            uint32_t* __restrict__ qweight) {
  const int chunks = (d + 31) / 32;
  const int nw = (int)(((long long)d * bits + 31) / 32);
  const long long item = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (item >= (long long)n * chunks) return;
  const int r = (int)(item / chunks), ch = (int)(item % chunks);
  const uint8_t* cr = codes + (long long)r * d + ch * 32;
  const int valid = min(32, d - ch * 32);
  const uint32_t mask = (1u << bits) - 1u;
  uint32_t* out = qweight + (long long)r * nw + ch * bits;
  uint64_t acc = 0;
  int nbits = 0, wi = 0;
  for (int k = 0; k < 32; ++k) {
    const uint32_t c = (k < valid) ? (cr[k] & mask) : 0u;
    acc |= (uint64_t)c << nbits;
    nbits += bits;
    if (nbits >= 32) {
      if (ch * bits + wi < nw) out[wi] = (uint32_t)acc;
      ++wi;
      acc >>= 32;
      nbits -= 32;
    }
  }
}

// Fast path for rows of whole 32-code chunks: one thread per chunk, the 32 codes in two 16-byte
// loads and the words in one 16-byte store (4 and 8 bits: two for 8), one 8-byte store (2 bits)
// or three word stores (3 bits). The host takes it only when codes is 16-byte aligned, d is a
// multiple of 32 and qweight is aligned for the store width, so every access is aligned.
template <int BITS>
__global__ void pack_vec_kernel(const uint8_t* __restrict__ codes, int n, int d,
                                uint32_t* __restrict__ qweight) {
  const long long item = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (item >= (long long)n * (d / 32)) return;
  const uint8_t* src;
  uint32_t* out;
  gptq::pack_chunk_ptrs<BITS>(codes, qweight, d, item, src, out);
  const uint4 a = __ldg(reinterpret_cast<const uint4*>(src));
  const uint4 b = __ldg(reinterpret_cast<const uint4*>(src) + 1);
  const uint32_t c[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  uint32_t w[BITS];
  gptq::pack32<BITS>(c, w);
  if constexpr (BITS == 4) {
    *reinterpret_cast<uint4*>(out) = make_uint4(w[0], w[1], w[2], w[3]);
  } else if constexpr (BITS == 8) {
    reinterpret_cast<uint4*>(out)[0] = make_uint4(w[0], w[1], w[2], w[3]);
    reinterpret_cast<uint4*>(out)[1] = make_uint4(w[4], w[5], w[6], w[7]);
  } else if constexpr (BITS == 2) {
    *reinterpret_cast<uint2*>(out) = make_uint2(w[0], w[1]);
  } else {
#pragma unroll
    for (int i = 0; i < BITS; ++i) out[i] = w[i];
  }
}

__global__ void to_f16_kernel(const float* __restrict__ a, const float* __restrict__ b,
                              uint16_t* __restrict__ ah, uint16_t* __restrict__ bh,
                              long long count) {
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < count;
       e += (long long)gridDim.x * blockDim.x) {
    ah[e] = __half_as_ushort(__float2half_rn(a[e]));
    bh[e] = __half_as_ushort(__float2half_rn(b[e]));
  }
}

inline int grid_cap(long long blocks) {
  const long long cap = (long long)gptq_host::num_sms() * 32;
  return (int)(blocks < 1 ? 1 : (blocks > cap ? cap : blocks));
}

}  // namespace

namespace gptq_host {

int rtn_launch(const void* W, int w_dtype, long long ldw, int n, int d, int bits, int group_size,
               int sym, uint8_t* codes, float* scales, float* zeros, cudaStream_t stream) {
  const int g = group_size > 0 ? group_size : d;
  const long long items = (long long)n * (d / g);
  const long long blocks = (items + 7) / 8;
  if (w_dtype == GPTQ_BF16)
    rtn_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(W), ldw, n, d, bits, g, sym, codes, scales, zeros);
  else
    rtn_kernel<float><<<(unsigned)blocks, 256, 0, stream>>>(static_cast<const float*>(W), ldw, n,
                                                            d, bits, g, sym, codes, scales, zeros);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int pack_launch(const uint8_t* codes, int n, int d, int bits, const float* scales,
                const float* zeros, long long n_groups, uint32_t* qweight, uint16_t* scales_f16,
                uint16_t* zeros_f16, cudaStream_t stream) {
  const long long items = (long long)n * ((d + 31) / 32);
  const unsigned blocks = (unsigned)((items + 255) / 256);
  const int store_align = bits == 2 ? 8 : (bits == 3 ? 4 : 16);
  const bool vec = d % 32 == 0 && (reinterpret_cast<uintptr_t>(codes) & 15) == 0 &&
                   (reinterpret_cast<uintptr_t>(qweight) & (uintptr_t)(store_align - 1)) == 0;
  if (vec && bits == 2)
    pack_vec_kernel<2><<<blocks, 256, 0, stream>>>(codes, n, d, qweight);
  else if (vec && bits == 3)
    pack_vec_kernel<3><<<blocks, 256, 0, stream>>>(codes, n, d, qweight);
  else if (vec && bits == 4)
    pack_vec_kernel<4><<<blocks, 256, 0, stream>>>(codes, n, d, qweight);
  else if (vec && bits == 8)
    pack_vec_kernel<8><<<blocks, 256, 0, stream>>>(codes, n, d, qweight);
  else
    pack_kernel<<<blocks, 256, 0, stream>>>(codes, n, d, bits, qweight);
  if (cudaGetLastError() != cudaSuccess) return GPTQ_ERR_CUDA;
  const long long cnt = (long long)n * n_groups;
  to_f16_kernel<<<grid_cap((cnt + 255) / 256), 256, 0, stream>>>(scales, zeros, scales_f16,
                                                                 zeros_f16, cnt);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

}  // namespace gptq_host
