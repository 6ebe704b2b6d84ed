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
// Layout: eight lanes own one row (four rows per warp); in each 32-column chunk of the block,
// lane s of a row holds the four contiguous columns 4s..4s+3, so one row of U is read with
// float4 loads, the remaining columns are spread evenly over the lanes, and chunks that are
// already quantized are skipped uniformly. For column j the owner lane evaluates the quantizer
// on its own value and broadcasts the error inside its 8-lane group; it keeps the code and the
// error in registers, and when a chunk is done every lane stores its four codes (one 32-bit
// word) and errors (one float4). The block's U (128 x 128, zero below the diagonal as
// gptq_prepare_hinv writes it) arrives in shared memory with one TMA copy; 1/U_jj is computed
// from it.
#include <float.h>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "gather4.cuh"
#include "pack32.cuh"
#include "kernels.h"
#include "tri_fill.cuh"

namespace {

constexpr int BLK = 128;
constexpr int ROWS_PER_WARP = 4;
constexpr int LANES_PER_ROW = 8;
static_assert(ROWS_PER_WARP * LANES_PER_ROW == 32, "eight lanes own one row");
constexpr int SW_SMEM = BLK * BLK * 4 + BLK * 4 + 64;
constexpr int SW_SMEM_STATIC = SW_SMEM + 3 * 16 * BLK * 4 + BLK * 4;  // + (s, 1/s, z) table

// q = clamp(rne(w / s) + z, 0, maxq) with the quotient rounded as in IEEE fp32 division, but
// formed as a multiplication by rs = 1/s (correctly rounded) wherever that cannot change the
// rounding. t = w * rs is within
// 3 * 2^-24 |w/s| (two roundings and the reciprocal's) of the correctly rounded quotient, so
// rint(t) equals rint(w / s) unless t lies within that distance of a rounding boundary
// (k + 1/2); only then is the quotient formed exactly. The margin used, 2^-21 |t|, covers the
// bound with room to spare.
// Lanes whose result is not used (exact = false) skip the exact quotient.
__device__ __forceinline__ float quant_code_rcp(float w, float s, float rs, float z, float maxq,
                                                bool exact = true) {
  float t = w * rs;
  float r = rintf(t);
  if (exact && fabsf(fabsf(t - r) - 0.5f) <= 4.76837158e-7f * fabsf(t)) r = rintf(__fdiv_rn(w, s));
  return fminf(fmaxf(r + z, 0.0f), maxq);
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

// Reductions over the eight lanes of a row group.
__device__ __forceinline__ float group8_min(float v) {
  v = fminf(v, __shfl_xor_sync(0xffffffffu, v, 1));
  v = fminf(v, __shfl_xor_sync(0xffffffffu, v, 2));
  return fminf(v, __shfl_xor_sync(0xffffffffu, v, 4));
}
__device__ __forceinline__ float group8_max(float v) {
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
  return fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
}

// (s, z, 1/s) of the group that starts at block column j, from the current values of its g
// columns (min / max over the row's eight lanes; w[4c + e] holds column 32c + 4 sub + e), and the
// stores of (s, z) (and their fp16 copies for the packed output) by the row's first lane.
__device__ __forceinline__ float3 group_params(const float (&w)[16], int j, int g, int sub,
                                               bool sym, int bits, float maxq, bool store,
                                               long long gi, float* scales, float* zeros,
                                               uint16_t* s16, uint16_t* z16) {
  float a = sym ? 0.f : FLT_MAX, b = -FLT_MAX, s, z;
#pragma unroll
  for (int c2 = 0; c2 < 4; ++c2)
#pragma unroll
    for (int e2 = 0; e2 < 4; ++e2) {
      const int k = 32 * c2 + 4 * sub + e2;
      const float v = w[4 * c2 + e2];
      if (k >= j && k < j + g) {
        if (sym) a = fmaxf(a, fabsf(v));
        else { a = fminf(a, v); b = fmaxf(b, v); }
      }
    }
  if (sym) {
    a = group8_max(a);
    sym_params(a, bits, s, z);
  } else {
    a = group8_min(a);
    b = group8_max(b);
    asym_params(a, b, maxq, s, z);
  }
  if (store) {
    scales[gi] = s;
    zeros[gi] = z;
    if (s16 != nullptr) {  // packed output: the fp16 copies (round to nearest even)
      s16[gi] = __half_as_ushort(__float2half_rn(s));
      z16[gi] = __half_as_ushort(__float2half_rn(z));
    }
  }
  return make_float3(s, z, __frcp_rn(s));
}

// 32 codes (c[i]: codes 4i .. 4i+3 as bytes) -> `bits` words of the packed row at out, the
// layout of gptq_pack (pack32.cuh). out is aligned for the vector store of each width: the row
// stride d * bits / 32 words and the chunk offset are multiples of it, qweight 16-byte aligned.
__device__ __forceinline__ void store_packed_chunk(const uint32_t (&c)[8], int bits,
                                                   uint32_t* out) {
  if (bits == 4) {
    uint32_t w[4];
    gptq::pack32<4>(c, w);
    *reinterpret_cast<uint4*>(out) = make_uint4(w[0], w[1], w[2], w[3]);
  } else if (bits == 3) {
    uint32_t w[3];
    gptq::pack32<3>(c, w);
    out[0] = w[0]; out[1] = w[1]; out[2] = w[2];
  } else if (bits == 2) {
    uint32_t w[2];
    gptq::pack32<2>(c, w);
    *reinterpret_cast<uint2*>(out) = make_uint2(w[0], w[1]);
  } else {
    uint32_t w[8];
    gptq::pack32<8>(c, w);
    reinterpret_cast<uint4*>(out)[0] = make_uint4(w[0], w[1], w[2], w[3]);
    reinterpret_cast<uint4*>(out)[1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
}

// STATIC: static groups (one instance each, so the default path carries no extra branch).
// FINE: groups shorter than 32 columns, whose starts fall inside a 32-column chunk.
template <bool STATIC, bool FINE>
__global__ void __launch_bounds__(128, 4)
sweep_block_kernel(const __grid_constant__ CUtensorMap tmap_u, const float* __restrict__ Wwork,
                   float* __restrict__ Err, uint8_t* __restrict__ codes,
                   float* __restrict__ scales, float* __restrict__ zeros, int n, int d, int col0,
                   int bits, int g, int sym, const int32_t* __restrict__ perm,
                   uint32_t* __restrict__ qweight, uint16_t* __restrict__ s16,
                   uint16_t* __restrict__ z16, int32_t* status) {
  extern __shared__ __align__(128) float sw_smem[];
  float* Us = sw_smem;                // [128][128], zero below the diagonal
  float* invd = sw_smem + BLK * BLK;  // [128]
  // Static groups: (s, 1/s, z) of every (row, column) of the block, [3][16][128], and the
  // original group of each column.
  float* stab = reinterpret_cast<float*>(sw_smem) + SW_SMEM / 4;
  int* sgid = reinterpret_cast<int*>(stab + 3 * 16 * BLK);
  uint64_t* bar = reinterpret_cast<uint64_t*>(invd + BLK);
  __shared__ int bad;
  __shared__ volatile int abort_flag;
  const int tid = threadIdx.x;
  if (tid == 0) {
    bad = gptq::status_bad(status) ? 1 : 0;
    abort_flag = 0;
    gptq::mbar_init(bar, 1);
    gptq::fence_barrier_init();
  }
  __syncthreads();
  if (bad) return;
  if (tid == 0) {
    gptq::mbar_arrive_expect_tx(bar, BLK * BLK * 4);
    gptq::tma_load_2d(Us, &tmap_u, bar, col0, col0);
  }
  // Meanwhile: this thread's row of W.
  const int warp = tid >> 5, lane = tid & 31;
  const int sub = lane & 7;                      // owns columns 32c + 4 sub + e
  const int grp = lane & ~7;                     // first lane of this row's group
  const int row = (blockIdx.x * (blockDim.x >> 5) + warp) * ROWS_PER_WARP + (lane >> 3);
  const bool live = row < n;
  const int rsafe = live ? row : 0;
  const float maxq = (float)((1 << bits) - 1);
  const int G = (g > 0) ? d / g : 1;
  const float* wrow = Wwork + (long long)rsafe * d + col0 + 4 * sub;
  float w[16];                                   // w[4c + e]: column 32c + 4 sub + e
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const float4 v = *reinterpret_cast<const float4*>(wrow + 32 * c);
    w[4 * c + 0] = v.x; w[4 * c + 1] = v.y; w[4 * c + 2] = v.z; w[4 * c + 3] = v.w;
  }
  float s = 1.f, z = 0.f;
  if (g <= 0) {  // one (s, z) per row, computed before the sweep
    s = scales[rsafe];
    z = zeros[rsafe];
  }
  float rs = __frcp_rn(s);
  if (STATIC) {  // parameters fixed before the sweep, looked up per column
    for (int t = tid; t < BLK; t += blockDim.x) sgid[t] = perm[col0 + t] / g;
    __syncthreads();
    for (int e = tid; e < 16 * BLK; e += blockDim.x) {
      const int r = blockIdx.x * 16 + e / BLK;
      const long long gi = (long long)(r < n ? r : n - 1) * G + sgid[e % BLK];
      const float sv = scales[gi];
      stab[e] = sv;
      stab[16 * BLK + e] = __frcp_rn(sv);
      stab[32 * BLK + e] = zeros[gi];
    }
  }
  const int rl = warp * ROWS_PER_WARP + (lane >> 3);  // this row within the CTA
  // Group sizes divide 128 and are multiples of 4, hence powers of two: a group starts where
  // the column's low bits are zero.
  const bool grouped = g > 0 && !STATIC;
  const int gmask = grouped ? g - 1 : 0;
  const bool landed = gptq::mbar_wait(bar, 0, &abort_flag);
  if (!__syncthreads_and(landed)) {  // the copy did not arrive in time: report, touch nothing
    if (tid == 0) {
      gptq::set_status(status, GPTQ_ERR_TIMEOUT, 3);
      gptq::mbar_drain(bar, 0);  // the CTA stays until the copy lands (bounded)
    }
    return;
  }
  for (int t = tid; t < BLK; t += blockDim.x) invd[t] = __fdiv_rn(1.0f, Us[t * BLK + t]);
  __syncthreads();

  float* erow = Err + (long long)rsafe * d + col0;
  uint8_t* crow = codes + (long long)rsafe * d + col0;
  const bool codes_vec = (reinterpret_cast<uintptr_t>(codes) & 3) == 0 && (d & 3) == 0;
  bool finite = true;
#pragma unroll
  for (int c = 0; c < 4; ++c) {                  // 32-column chunks
    float qk[4], ek[4];                          // this lane's four codes and errors of chunk c
    // Groups of 32 columns or more start at chunk starts: their statistics are taken here,
    // outside the column loop (which keeps that loop's unrolled code small).
    if (!FINE && grouped && ((32 * c) & gmask) == 0) {
      const float3 p = group_params(w, 32 * c, g, sub, sym, bits, maxq, sub == 0 && live,
                                    (long long)row * G + (col0 + 32 * c) / g, scales, zeros,
                                    s16, z16);
      s = p.x; z = p.y; rs = p.z;
    }
    // Columns 32c + 4 so + e: lane so of the row's group owns the four of a run. Every lane
    // quantizes its own slot (only the owner's result is kept), so the owner needs no broadcast
    // to decide a column; the error is then broadcast for the other lanes' updates. The owner
    // forms its next column's value from its own error, and that next decision is written
    // before this column's updates, which wait on the broadcast: issue is in order, so the
    // decisions of a run follow one another without the broadcast in between. Only the step to
    // the next lane's run waits on it. (Groups shorter than 32 columns take their statistics
    // inside the run from every lane's updated values, so that case keeps the plain order.)
#pragma unroll 1
    for (int so = 0; so < 8; ++so) {             // owner sub-lane within the chunk
      const bool owner = sub == so;
      const int j0 = 32 * c + 4 * so;
      if (STATIC) {
        s = stab[rl * BLK + j0];
        rs = stab[16 * BLK + rl * BLK + j0];
        z = stab[32 * BLK + rl * BLK + j0];
      } else if (FINE && (j0 & gmask) == 0) {
        const float3 p = group_params(w, j0, g, sub, sym, bits, maxq, sub == 0 && live,
                                      (long long)row * G + (col0 + j0) / g, scales, zeros, s16,
                                      z16);
        s = p.x; z = p.y; rs = p.z;
      }
      float xcur = w[4 * c];                     // the owner's column j0, up to date
      float qv = quant_code_rcp(xcur, s, rs, z, maxq, owner);
      float eo = (xcur - s * (qv - z)) * invd[j0];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = j0 + e;
        const float err = __shfl_sync(0xffffffffu, eo, grp | so);
        if (owner) {
          qk[e] = qv;
          ek[e] = eo;
        }
        finite = finite && (fabsf(err) <= FLT_MAX);
        const float* urow = Us + j * BLK + 4 * sub;
        const float4 uc = *reinterpret_cast<const float4*>(urow + 32 * c);
        float qn = 0.f, en = 0.f;
        if (!FINE && e < 3) {
          // column j + 1: the owner's value from its own error, decided before the updates
          const float un = e == 0 ? uc.y : (e == 1 ? uc.z : uc.w);
          const float xn = fmaf(-eo, un, w[4 * c + e + 1]);
          if (STATIC) {
            s = stab[rl * BLK + j + 1];
            rs = stab[16 * BLK + rl * BLK + j + 1];
            z = stab[32 * BLK + rl * BLK + j + 1];
          }
          qn = quant_code_rcp(xn, s, rs, z, maxq, owner);
          en = (xn - s * (qn - z)) * invd[j + 1];
        }
        // w_k -= err * U_jk for the columns of chunks c..3 (U_jk = 0 for k < j).
        w[4 * c + 0] = fmaf(-err, uc.x, w[4 * c + 0]);
        w[4 * c + 1] = fmaf(-err, uc.y, w[4 * c + 1]);
        w[4 * c + 2] = fmaf(-err, uc.z, w[4 * c + 2]);
        w[4 * c + 3] = fmaf(-err, uc.w, w[4 * c + 3]);
#pragma unroll
        for (int c2 = c + 1; c2 < 4; ++c2) {
          const float4 u = *reinterpret_cast<const float4*>(urow + 32 * c2);
          w[4 * c2 + 0] = fmaf(-err, u.x, w[4 * c2 + 0]);
          w[4 * c2 + 1] = fmaf(-err, u.y, w[4 * c2 + 1]);
          w[4 * c2 + 2] = fmaf(-err, u.z, w[4 * c2 + 2]);
          w[4 * c2 + 3] = fmaf(-err, u.w, w[4 * c2 + 3]);
        }
        if (e < 3) {
          if (FINE) {  // plain order: statistics (at a group start) and decision after updates
            const int jn = j + 1;
            if ((jn & gmask) == 0) {
              const float3 p = group_params(w, jn, g, sub, sym, bits, maxq, sub == 0 && live,
                                            (long long)row * G + (col0 + jn) / g, scales, zeros,
                                            s16, z16);
              s = p.x; z = p.y; rs = p.z;
            }
            xcur = w[4 * c + e + 1];
            qn = quant_code_rcp(xcur, s, rs, z, maxq, owner);
            en = (xcur - s * (qn - z)) * invd[jn];
          }
          qv = qn;
          eo = en;
        }
      }
    }
    // Chunk done: each lane stores its four columns 32c + 4 sub .. +3 at once.
    if (live) {
      const int k0 = 32 * c + 4 * sub;
      *reinterpret_cast<float4*>(erow + k0) = make_float4(ek[0], ek[1], ek[2], ek[3]);
    }
    const uint32_t packed = (uint32_t)qk[0] | ((uint32_t)qk[1] << 8) | ((uint32_t)qk[2] << 16) |
                            ((uint32_t)qk[3] << 24);
    if (qweight != nullptr) {
      // Packed output: the row's 32 codes of this chunk (four per lane) gathered in every lane
      // of the row's group, packed by its first lane into `bits` words of the row's bit stream.
      uint32_t cw[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) cw[k] = __shfl_sync(0xffffffffu, packed, grp | k);
      if (sub == 0 && live)
        store_packed_chunk(cw, bits, qweight + (long long)row * (d / 32) * bits +
                                         (long long)(col0 / 32 + c) * bits);
    } else if (live) {
      const int k0 = 32 * c + 4 * sub;
      if (codes_vec) {
        *reinterpret_cast<uint32_t*>(crow + k0) = packed;
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) crow[k0 + e] = (uint8_t)(packed >> (8 * e));
      }
    }
  }
  if (!finite && live) gptq::set_status(status, GPTQ_ERR_NONFINITE, col0);
}

// Wwork[r][k] = dead[k] ? 0 : W[r][perm[k]] as fp32 (bf16 widened exactly). A thread owns four
// consecutive columns (d is a multiple of 128): their sources and liveness are read once, then
// for each of its rows (blockIdx.y, grid-stride) four loads and one 16-byte store.
template <typename T>  // float, or uint16_t holding bf16 bit patterns
__global__ void gather_w_kernel(const T* __restrict__ W, long long ldw, int n, int d,
                                const int32_t* __restrict__ perm, const uint8_t* __restrict__ dead,
                                float* __restrict__ Wwork, const int32_t* status) {
  if (gptq::status_bad(status)) return;
  const int k0 = 4 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (k0 >= d) return;
  int32_t src[4];
  bool live[4];
  gptq::gather4_cols(perm, dead, k0, src, live);
  for (long long r = blockIdx.y; r < n; r += gridDim.y) {
    float v[4];
    gptq::gather4_row<T>(W, ldw, r, src, live, v);
    *reinterpret_cast<float4*>(Wwork + r * d + k0) = make_float4(v[0], v[1], v[2], v[3]);
  }
}

// One (s, z) per row from the whole row at the start of the sweep (group_size = -1).
__global__ void row_params_kernel(const float* __restrict__ Wwork, int n, int d, int bits,
                                  int sym, float* __restrict__ scales,
                                  float* __restrict__ zeros, uint16_t* __restrict__ s16,
                                  uint16_t* __restrict__ z16, const int32_t* status) {
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
    if (s16 != nullptr) {
      s16[r] = __half_as_ushort(__float2half_rn(s));
      z16[r] = __half_as_ushort(__float2half_rn(z));
    }
  }
}

__global__ void unpermute_codes_kernel(const uint8_t* __restrict__ cs,
                                       const int32_t* __restrict__ perm,
                                       uint8_t* __restrict__ codes, int n, int d,
                                       const int32_t* status) {
  if (gptq::status_bad(status)) return;
  // Rows on grid y, columns strided over grid x (tri_fill.cuh): no per-element division.
  for (long long r = blockIdx.y; r < n; r += gridDim.y) {
    long long lo, hi;
    gptq::tri_row_span(gptq::kWholeRow, r, d, lo, hi);
    for (long long k = lo + blockIdx.x * (long long)blockDim.x + threadIdx.x; k < hi;
         k += (long long)gridDim.x * blockDim.x)
      gptq::unpermute_elem(cs, perm, codes, d, r, k);
  }
}

// Permuted column order, packed output: one thread per (row, chunk of 32 original columns)
// gathers its codes from the sweep-order codes (original column c sits at sweep position
// inv[c]) and packs them into `bits` words (pack32.cuh). d is a multiple of 128.
template <int BITS>
__global__ void unpermute_pack_kernel(const uint8_t* __restrict__ cs,
                                      const int32_t* __restrict__ inv, int n, int d,
                                      uint32_t* __restrict__ qweight, const int32_t* status) {
  if (gptq::status_bad(status)) return;
  const int chunks = d / 32;
  for (long long item = blockIdx.x * (long long)blockDim.x + threadIdx.x;
       item < (long long)n * chunks; item += (long long)gridDim.x * blockDim.x) {
    const long long r = item / chunks;
    const int ch = (int)(item % chunks);
    const uint8_t* row = cs + r * d;
    uint32_t c[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      uint32_t v = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) v |= (uint32_t)row[inv[ch * 32 + 4 * i + e]] << (8 * e);
      c[i] = v;
    }
    store_packed_chunk(c, BITS, qweight + r * chunks * BITS + (long long)ch * BITS);
  }
}

// g_idx[perm[k]] = k / g (groups in sweep order); perm == nullptr: g_idx[k] = k / g.
__global__ void g_idx_kernel(const int32_t* __restrict__ perm, int32_t* __restrict__ g_idx, int d,
                             int g, const int32_t* status) {
  if (gptq::status_bad(status)) return;
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < d; k += gridDim.x * blockDim.x)
    g_idx[perm ? perm[k] : k] = (g > 0) ? k / g : 0;
}

// inv[perm[j]] = j.
__global__ void invert_perm_kernel(const int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                                   int d, const int32_t* status) {
  if (gptq::status_bad(status)) return;
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < d; j += gridDim.x * blockDim.x)
    inv[perm[j]] = j;
}

// Static groups: (s, z) of each run of g columns in the original order, from the working copy
// (sweep order, dead columns zero; original column c sits at sweep position inv[c]). One warp
// per row; the lanes take the group's columns in turn.
__global__ void static_params_kernel(const float* __restrict__ Wwork,
                                     const int32_t* __restrict__ inv, int n, int d, int g,
                                     int bits, int sym, float* __restrict__ scales,
                                     float* __restrict__ zeros, uint16_t* __restrict__ s16,
                                     uint16_t* __restrict__ z16, const int32_t* status) {
  if (gptq::status_bad(status)) return;
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= n) return;
  const float* wr = Wwork + (long long)r * d;
  const int G = d / g;
  const float maxq = (float)((1 << bits) - 1);
  for (int q = 0; q < G; ++q) {
    float mn = FLT_MAX, mx = -FLT_MAX, am = 0.f;
    for (int c = q * g + lane; c < q * g + g; c += 32) {
      const float v = wr[inv[c]];
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
      float sv, zv;
      if (sym) sym_params(am, bits, sv, zv);
      else asym_params(mn, mx, maxq, sv, zv);
      scales[(long long)r * G + q] = sv;
      zeros[(long long)r * G + q] = zv;
      if (s16 != nullptr) {
        s16[(long long)r * G + q] = __half_as_ushort(__float2half_rn(sv));
        z16[(long long)r * G + q] = __half_as_ushort(__float2half_rn(zv));
      }
    }
  }
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
  // d is a multiple of 128 and Wwork 16-byte aligned (checked by the entry point), so every
  // thread's four columns exist and its float4 store is aligned.
  const dim3 grid((unsigned)((d / 4 + 255) / 256), (unsigned)(n < 65535 ? n : 65535));
  if (w_dtype == GPTQ_BF16)
    gather_w_kernel<uint16_t><<<grid, 256, 0, stream>>>(static_cast<const uint16_t*>(W), ldw, n,
                                                        d, perm, dead, Wwork, status);
  else
    gather_w_kernel<float><<<grid, 256, 0, stream>>>(static_cast<const float*>(W), ldw, n, d,
                                                     perm, dead, Wwork, status);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int sweep_row_params(const float* Wwork, int n, int d, int bits, int sym, float* scales,
                     float* zeros, uint16_t* s16, uint16_t* z16, const int32_t* status,
                     cudaStream_t stream) {
  row_params_kernel<<<(n + 7) / 8, 256, 0, stream>>>(Wwork, n, d, bits, sym, scales, zeros, s16,
                                                     z16, status);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int sweep_block(float* Wwork, const float* U, float* Err, uint8_t* codes, float* scales,
                float* zeros, int n, int d, int col0, int bits, int group_size, int sym,
                const int32_t* perm, int static_groups, uint32_t* qweight, uint16_t* s16,
                uint16_t* z16, int32_t* status, cudaStream_t stream) {
  if (ensure_smem_attr(reinterpret_cast<const void*>(sweep_block_kernel<false, false>), SW_SMEM) !=
          0 ||
      ensure_smem_attr(reinterpret_cast<const void*>(sweep_block_kernel<false, true>), SW_SMEM) !=
          0 ||
      ensure_smem_attr(reinterpret_cast<const void*>(sweep_block_kernel<true, false>),
                       SW_SMEM_STATIC) != 0)
    return GPTQ_ERR_CUDA;
  CUtensorMap tu;  // the whole U (d x d fp32), copied 128 x 128 at a time without swizzle
  if (make_tmap_2d(&tu, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, U, (uint64_t)d, (uint64_t)d,
                   (uint64_t)d * 4, BLK, BLK, CU_TENSOR_MAP_SWIZZLE_NONE) != 0)
    return GPTQ_ERR_CUDA;
  const int warps_total = (n + ROWS_PER_WARP - 1) / ROWS_PER_WARP;
  const int grid = (warps_total + 3) / 4;  // 4 warps (16 rows) per CTA
  if (static_groups)
    sweep_block_kernel<true, false><<<grid, 128, SW_SMEM_STATIC, stream>>>(
        tu, Wwork, Err, codes, scales, zeros, n, d, col0, bits, group_size, sym, perm, qweight,
        s16, z16, status);
  else if (group_size > 0 && group_size < 32)
    sweep_block_kernel<false, true><<<grid, 128, SW_SMEM, stream>>>(
        tu, Wwork, Err, codes, scales, zeros, n, d, col0, bits, group_size, sym, perm, qweight,
        s16, z16, status);
  else
    sweep_block_kernel<false, false><<<grid, 128, SW_SMEM, stream>>>(
        tu, Wwork, Err, codes, scales, zeros, n, d, col0, bits, group_size, sym, perm, qweight,
        s16, z16, status);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int sweep_unpermute_codes(const uint8_t* codes_sweep, const int32_t* perm, uint8_t* codes, int n,
                          int d, const int32_t* status, cudaStream_t stream) {
  const dim3 grid((unsigned)((d + 1023) / 1024), (unsigned)(n < 65535 ? n : 65535));
  unpermute_codes_kernel<<<grid, 256, 0, stream>>>(codes_sweep, perm, codes, n, d, status);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int sweep_invert_perm(const int32_t* perm, int32_t* inv, int d, const int32_t* status,
                      cudaStream_t stream) {
  invert_perm_kernel<<<grid_for(d), 256, 0, stream>>>(perm, inv, d, status);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int sweep_static_params(const float* Wwork, const int32_t* inv, int n, int d, int group_size,
                        int bits, int sym, float* scales, float* zeros, uint16_t* s16,
                        uint16_t* z16, const int32_t* status, cudaStream_t stream) {
  static_params_kernel<<<(n + 7) / 8, 256, 0, stream>>>(Wwork, inv, n, d, group_size, bits, sym,
                                                         scales, zeros, s16, z16, status);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int sweep_unpermute_pack(const uint8_t* codes_sweep, const int32_t* inv, int n, int d, int bits,
                         uint32_t* qweight, const int32_t* status, cudaStream_t stream) {
  const long long items = (long long)n * (d / 32);
  const int grid = grid_for(items);
  if (bits == 2)
    unpermute_pack_kernel<2><<<grid, 256, 0, stream>>>(codes_sweep, inv, n, d, qweight, status);
  else if (bits == 3)
    unpermute_pack_kernel<3><<<grid, 256, 0, stream>>>(codes_sweep, inv, n, d, qweight, status);
  else if (bits == 4)
    unpermute_pack_kernel<4><<<grid, 256, 0, stream>>>(codes_sweep, inv, n, d, qweight, status);
  else
    unpermute_pack_kernel<8><<<grid, 256, 0, stream>>>(codes_sweep, inv, n, d, qweight, status);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int sweep_g_idx(const int32_t* perm, int32_t* g_idx, int d, int group_size,
                const int32_t* status, cudaStream_t stream) {
  g_idx_kernel<<<grid_for(d), 256, 0, stream>>>(perm, g_idx, d, group_size, status);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

}  // namespace gptq_host
