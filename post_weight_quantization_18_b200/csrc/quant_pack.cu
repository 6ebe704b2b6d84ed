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
// fill exactly b words.
#include <float.h>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"

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
  pack_kernel<<<(unsigned)((items + 255) / 256), 256, 0, stream>>>(codes, n, d, bits, qweight);
  if (cudaGetLastError() != cudaSuccess) return GPTQ_ERR_CUDA;
  const long long cnt = (long long)n * n_groups;
  to_f16_kernel<<<grid_cap((cnt + 255) / 256), 256, 0, stream>>>(scales, zeros, scales_f16,
                                                                 zeros_f16, cnt);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

}  // namespace gptq_host
