// sweep.cu — the GPTQ column sweep of one 128-column block, and its prologue / epilogue.
//
// "GPTQ: Mathematical Foundations ...", §1 Arbitrary Order Quantization (one fixed column
// order for all rows), §2 Lazy Batch Updates (inside a block of B = 128 columns each quantized
// column immediately updates the block's later columns), §3 Cholesky Decomposition (the
// compensation of column k by column j is U_jk / U_jj with H^-1 = U^T U); "INT4 and GPTQ
// Quantization", §The GPTQ Update Rule and §Group Quantization.
//
// For column j of a row:  q = clamp(rne(w_j / s) + z, 0, 2^b - 1),  w_hat = s (q - z),
//                         err_j = (w_j - w_hat) / U_jj,  w_k -= err_j U_jk (k > j in block).
// (s, z) of a group are taken when the sweep reaches the group's first column, from the
// current (compensated) values of its g columns; with one scale per row they come from the
// row at the start of the sweep (sweep_row_params).
//
// Layout: one warp owns two rows (two independent dependency chains); lane l holds columns
// 4l..4l+3 of each row in registers. Every lane evaluates the quantizer for column j on the
// value broadcast from its owner lane, so no second broadcast is needed; the block's U
// (128 x 128, zero below the diagonal) and 1/U_jj are staged in shared memory.
#include <float.h>

#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace {

constexpr int BLK = 128;
constexpr int SW_THREADS = 256;
constexpr int RPW = 2;                                   // rows per warp
constexpr int ROWS_PER_CTA = (SW_THREADS / 32) * RPW;    // 16
constexpr int SW_SMEM = BLK * BLK * 4 + BLK * 4;

__device__ __forceinline__ float quant_code(float w, float s, float z, float maxq) {
  const float q = rintf(__fdiv_rn(w, s)) + z;
  return fminf(fmaxf(q, 0.0f), maxq);
}

__device__ __forceinline__ void asym_params(float mn, float mx, float maxq, float& s, float& z) {
  s = __fdiv_rn(mx - mn, maxq);
  if (s == 0.0f) s = 1.0f;
  z = fminf(fmaxf(rintf(__fdiv_rn(-mn, s)), 0.0f), maxq);
}

__device__ __forceinline__ void sym_params(float amax, int bits, float& s, float& z) {
  s = __fdiv_rn(amax, (float)((1 << (bits - 1)) - 1));
  if (s == 0.0f) s = 1.0f;
  z = (float)(1 << (bits - 1));
}

__global__ void __launch_bounds__(SW_THREADS)
sweep_block_kernel(const float* __restrict__ Wwork, const float* __restrict__ U,
                   float* __restrict__ Err, uint8_t* __restrict__ codes,
                   float* __restrict__ scales, float* __restrict__ zeros, int n, int d, int col0,
                   int bits, int g, int sym, int32_t* status) {
  extern __shared__ __align__(16) float sw_smem[];
  float* Us = sw_smem;               // [128][128]
  float* invd = sw_smem + BLK * BLK;  // [128]
  __shared__ int bad;
  const int tid = threadIdx.x;
  if (tid == 0) bad = gptq::status_bad(status) ? 1 : 0;
  // Stage U[col0 .. col0+127][col0 .. col0+127] (entries below the diagonal forced to zero).
  for (int e = tid; e < BLK * (BLK / 4); e += SW_THREADS) {
    const int r = e / (BLK / 4), c4 = e % (BLK / 4);
    float4 v = *reinterpret_cast<const float4*>(U + (long long)(col0 + r) * d + col0 + 4 * c4);
    if (4 * c4 + 0 < r) v.x = 0.f;
    if (4 * c4 + 1 < r) v.y = 0.f;
    if (4 * c4 + 2 < r) v.z = 0.f;
    if (4 * c4 + 3 < r) v.w = 0.f;
    *reinterpret_cast<float4*>(Us + r * BLK + 4 * c4) = v;
  }
  if (tid < BLK) invd[tid] = __fdiv_rn(1.0f, U[(long long)(col0 + tid) * d + col0 + tid]);
  __syncthreads();
  if (bad) return;

  const int warp = tid >> 5, lane = tid & 31;
  const float maxq = (float)((1 << bits) - 1);
  const int G = (g > 0) ? d / g : 1;
  int row[RPW];
  bool live[RPW];
  float w[RPW][4], errv[RPW][4];
  uint32_t cpack[RPW];
  float s[RPW], z[RPW];
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    row[rr] = blockIdx.x * ROWS_PER_CTA + warp * RPW + rr;
    live[rr] = row[rr] < n;
    const int rsafe = live[rr] ? row[rr] : 0;
    const float4 v =
        *reinterpret_cast<const float4*>(Wwork + (long long)rsafe * d + col0 + 4 * lane);
    w[rr][0] = v.x; w[rr][1] = v.y; w[rr][2] = v.z; w[rr][3] = v.w;
    cpack[rr] = 0u;
    errv[rr][0] = errv[rr][1] = errv[rr][2] = errv[rr][3] = 0.f;
    if (g <= 0) {  // one (s, z) per row, computed before the sweep
      s[rr] = scales[rsafe];
      z[rr] = zeros[rsafe];
    } else {
      s[rr] = 1.f;
      z[rr] = 0.f;
    }
  }

#pragma unroll 1
  for (int l = 0; l < 32; ++l) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int j = 4 * l + c;
      if (g > 0 && (j % g) == 0) {
        // Group [j, j+g): lanes j/4 .. (j+g)/4 - 1 hold its columns.
        const bool in_grp = (4 * lane >= j) && (4 * lane < j + g);
#pragma unroll
        for (int rr = 0; rr < RPW; ++rr) {
          float a, b;
          if (sym) {
            a = in_grp ? fmaxf(fmaxf(fabsf(w[rr][0]), fabsf(w[rr][1])),
                               fmaxf(fabsf(w[rr][2]), fabsf(w[rr][3])))
                       : 0.f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
            sym_params(a, bits, s[rr], z[rr]);
          } else {
            a = in_grp ? fminf(fminf(w[rr][0], w[rr][1]), fminf(w[rr][2], w[rr][3])) : FLT_MAX;
            b = in_grp ? fmaxf(fmaxf(w[rr][0], w[rr][1]), fmaxf(w[rr][2], w[rr][3])) : -FLT_MAX;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
              a = fminf(a, __shfl_xor_sync(0xffffffffu, a, o));
              b = fmaxf(b, __shfl_xor_sync(0xffffffffu, b, o));
            }
            asym_params(a, b, maxq, s[rr], z[rr]);
          }
          if (lane == 0 && live[rr]) {
            const long long gi = (long long)row[rr] * G + (col0 + j) / g;
            scales[gi] = s[rr];
            zeros[gi] = z[rr];
          }
        }
      }
      const float4 u4 = *reinterpret_cast<const float4*>(Us + j * BLK + 4 * lane);
      const float id = invd[j];
#pragma unroll
      for (int rr = 0; rr < RPW; ++rr) {
        const float wj = __shfl_sync(0xffffffffu, w[rr][c], l);
        const float q = quant_code(wj, s[rr], z[rr], maxq);
        const float wh = s[rr] * (q - z[rr]);
        const float err = (wj - wh) * id;
        if (lane == l) {
          cpack[rr] |= ((uint32_t)q) << (8 * c);
          errv[rr][c] = err;
        }
        w[rr][0] = fmaf(-err, u4.x, w[rr][0]);
        w[rr][1] = fmaf(-err, u4.y, w[rr][1]);
        w[rr][2] = fmaf(-err, u4.z, w[rr][2]);
        w[rr][3] = fmaf(-err, u4.w, w[rr][3]);
      }
    }
  }

  bool finite = true;
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    if (!live[rr]) continue;
    *reinterpret_cast<uint32_t*>(codes + (long long)row[rr] * d + col0 + 4 * lane) = cpack[rr];
    *reinterpret_cast<float4*>(Err + (long long)row[rr] * d + col0 + 4 * lane) =
        make_float4(errv[rr][0], errv[rr][1], errv[rr][2], errv[rr][3]);
#pragma unroll
    for (int c = 0; c < 4; ++c) finite = finite && (fabsf(errv[rr][c]) <= FLT_MAX);
  }
  if (!finite) gptq::set_status(status, GPTQ_ERR_NONFINITE, col0);
}

// Wwork[r][k] = dead[k] ? 0 : W[r][perm[k]] as fp32 (bf16 widened exactly).
template <typename T>
__global__ void gather_w_kernel(const T* __restrict__ W, long long ldw, int n, int d,
                                const int32_t* __restrict__ perm, const uint8_t* __restrict__ dead,
                                float* __restrict__ Wwork, const int32_t* status) {
  if (gptq::status_bad(status)) return;
  const long long total = (long long)n * d;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(e / d), k = (int)(e % d);
    float v = 0.f;
    if (!dead[k]) {
      if constexpr (sizeof(T) == 2)
        v = __bfloat162float(W[(long long)r * ldw + perm[k]]);
      else
        v = W[(long long)r * ldw + perm[k]];
    }
    Wwork[e] = v;
  }
}

// One (s, z) per row from the whole row at the start of the sweep (group_size = -1).
__global__ void row_params_kernel(const float* __restrict__ Wwork, int n, int d, int bits,
                                  int sym, float* __restrict__ scales,
                                  float* __restrict__ zeros, const int32_t* status) {
  if (gptq::status_bad(status)) return;
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= n) return;
  float mn = FLT_MAX, mx = -FLT_MAX, am = 0.f;
  for (int k = lane; k < d; k += 32) {
    const float v = Wwork[(long long)r * d + k];
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
  if (lane == 0) {
    float s, z;
    if (sym) sym_params(am, bits, s, z);
    else asym_params(mn, mx, (float)((1 << bits) - 1), s, z);
    scales[r] = s;
    zeros[r] = z;
  }
}

__global__ void unpermute_codes_kernel(const uint8_t* __restrict__ cs,
                                       const int32_t* __restrict__ perm,
                                       uint8_t* __restrict__ codes, int n, int d,
                                       const int32_t* status) {
  if (gptq::status_bad(status)) return;
  const long long total = (long long)n * d;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(e / d), k = (int)(e % d);
    codes[(long long)r * d + perm[k]] = cs[e];
  }
}

__global__ void g_idx_kernel(const int32_t* __restrict__ perm, int32_t* __restrict__ g_idx, int d,
                             int g) {
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < d; k += gridDim.x * blockDim.x)
    g_idx[perm[k]] = (g > 0) ? k / g : 0;
}

inline int grid_for(long long total) {
  long long gr = (total + 255) / 256;
  const long long cap = (long long)gptq_host::num_sms() * 16;
  return (int)(gr < 1 ? 1 : (gr > cap ? cap : gr));
}

}  // namespace

namespace gptq_host {

int sweep_gather_w(const void* W, int w_dtype, long long ldw, int n, int d, const int32_t* perm,
                   const uint8_t* dead, float* Wwork, const int32_t* status,
                   cudaStream_t stream) {
  const int gr = grid_for((long long)n * d);
  if (w_dtype == GPTQ_BF16)
    gather_w_kernel<__nv_bfloat16><<<gr, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(W), ldw, n, d, perm, dead, Wwork, status);
  else
    gather_w_kernel<float><<<gr, 256, 0, stream>>>(static_cast<const float*>(W), ldw, n, d, perm,
                                                   dead, Wwork, status);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int sweep_row_params(const float* Wwork, int n, int d, int bits, int sym, float* scales,
                     float* zeros, const int32_t* status, cudaStream_t stream) {
  row_params_kernel<<<(n + 7) / 8, 256, 0, stream>>>(Wwork, n, d, bits, sym, scales, zeros,
                                                     status);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int sweep_block(float* Wwork, const float* U, float* Err, uint8_t* codes, float* scales,
                float* zeros, int n, int d, int col0, int bits, int group_size, int sym,
                int32_t* status, cudaStream_t stream) {
  if (cudaFuncSetAttribute(sweep_block_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           SW_SMEM) != cudaSuccess)
    return GPTQ_ERR_CUDA;
  const int grid = (n + ROWS_PER_CTA - 1) / ROWS_PER_CTA;
  sweep_block_kernel<<<grid, SW_THREADS, SW_SMEM, stream>>>(Wwork, U, Err, codes, scales, zeros,
                                                            n, d, col0, bits, group_size, sym,
                                                            status);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int sweep_unpermute_codes(const uint8_t* codes_sweep, const int32_t* perm, uint8_t* codes, int n,
                          int d, const int32_t* status, cudaStream_t stream) {
  unpermute_codes_kernel<<<grid_for((long long)n * d), 256, 0, stream>>>(codes_sweep, perm,
                                                                         codes, n, d, status);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int sweep_g_idx(const int32_t* perm, int32_t* g_idx, int d, int group_size, cudaStream_t stream) {
  g_idx_kernel<<<grid_for(d), 256, 0, stream>>>(perm, g_idx, d, group_size);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

}  // namespace gptq_host
