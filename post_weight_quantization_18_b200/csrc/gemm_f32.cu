// gemm_f32.cu — C = alpha * op(A) op(B) + beta * C in fp32 (row-major) on CUDA cores, and the
// dispatcher gemm_f32() that routes every fp32 product of the library.
//
// Serves the fp32 pieces of the path: the lazy trailing update W[:, F] -= Err_B U[B, F]
// ("GPTQ: Mathematical Foundations ...", §2 Lazy Batch Updates), the GEMM steps of the
// Cholesky / triangular-inverse schedule, and the Hessian of fp32 calibration inputs.
//   gemm_f32_staged_kernel  products up to 512 x 512 x 512 (the critical chain of prepare and
//                           the sweep's small updates): 32 x 32 (or 64 x 32) output tile per
//                           CTA, the tile's whole k-range staged with one round of 16-byte
//                           loads, split over the warps, partial sums added in shared memory.
//   gemm_f32_small_kernel   other small outputs (up to 4 tiles of 128 x 128).
//   gemm_f32_simt_kernel    operands TMA cannot address: 128 x 128 tile per 256-thread CTA,
//                           8 x 8 outputs per thread, k-slabs of 16 staged in shared memory.
// Everything else goes to the tcgen05 3xTF32 kernel (gemm_tf32x3.cu).
#include "common.cuh"
#include "kernels.h"

namespace {

constexpr int TM = 128, TN = 128, TK = 16, THREADS = 256;

__global__ void __launch_bounds__(THREADS)
gemm_f32_simt_kernel(int M, int N, int K, float alpha, const float* __restrict__ A, long long lda,
                     int transA, const float* __restrict__ B, long long ldb, int transB,
                     float beta, float* __restrict__ C, long long ldc, int upper_only,
                     int tri, const int32_t* status) {
  __shared__ __align__(16) float As[2][TK][TM + 4];
  __shared__ __align__(16) float Bs[2][TK][TN + 4];
  if (gptq::status_bad(status)) return;
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
  if (upper_only && m0 > n0 + TN - 1) return;  // tile entirely below the diagonal
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;

  auto load = [&](int buf, int k0) {
    // A slab: op(A)[m0 + mm][k0 + kk], 128 x 16 = 2048 values, 8 per thread.
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int e = tid + r * THREADS;
      int mm, kk;
      if (transA) { mm = e & (TM - 1); kk = e >> 7; }   // consecutive threads along m
      else { kk = e & (TK - 1); mm = e >> 4; }          // consecutive threads along k
      const int gm = m0 + mm, gk = k0 + kk;
      float v = 0.f;
      if (gm < M && gk < K) v = transA ? A[(long long)gk * lda + gm] : A[(long long)gm * lda + gk];
      As[buf][kk][mm] = v;
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int e = tid + r * THREADS;
      int nn, kk;
      if (!transB) { nn = e & (TN - 1); kk = e >> 7; }
      else { kk = e & (TK - 1); nn = e >> 4; }
      const int gn = n0 + nn, gk = k0 + kk;
      float v = 0.f;
      if (gn < N && gk < K) v = transB ? B[(long long)gn * ldb + gk] : B[(long long)gk * ldb + gn];
      Bs[buf][kk][nn] = v;
    }
  };

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  int k_lo, k_hi;
  gptq_host::tri_k_range(tri, m0, n0, n0 + TN, K, k_lo, k_hi);
  const int kt0 = k_lo / TK, nk = (k_hi + TK - 1) / TK;
  if (kt0 < nk) load(0, kt0 * TK);
  __syncthreads();
  for (int kt = kt0; kt < nk; ++kt) {
    const int cur = (kt - kt0) & 1;
    if (kt + 1 < nk) load(cur ^ 1, (kt + 1) * TK);
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[8], b[8];
      const float4 a0 = *reinterpret_cast<const float4*>(&As[cur][kk][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[cur][kk][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[cur][kk][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[cur][kk][64 + tx * 4]);
      a[0] = a0.x; a[1] = a0.y; a[2] = a0.z; a[3] = a0.w;
      a[4] = a1.x; a[5] = a1.y; a[6] = a1.z; a[7] = a1.w;
      b[0] = b0.x; b[1] = b0.y; b[2] = b0.z; b[3] = b0.w;
      b[4] = b1.x; b[5] = b1.y; b[6] = b1.z; b[7] = b1.w;
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int gm = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int gn = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4));
      if (gn >= N) continue;
      if (upper_only && gm > gn) continue;
      float* cp = C + (long long)gm * ldc + gn;
      const float v = alpha * acc[i][j];
      *cp = (beta == 0.f) ? v : fmaf(beta, *cp, v);
    }
  }
}

// Small GEMMs (the bottom levels of the recursions): 32 x 32 output tiles so that even a
// 128 x 128 product spreads over 16 CTAs; 256 threads, 2 x 2 outputs each, 32-deep k-slabs.
constexpr int ST = 32, SK = 32;

__global__ void __launch_bounds__(256)
gemm_f32_small_kernel(int M, int N, int K, float alpha, const float* __restrict__ A, long long lda,
                      int transA, const float* __restrict__ B, long long ldb, int transB,
                      float beta, float* __restrict__ C, long long ldc, int upper_only,
                      int tri, const int32_t* status) {
  __shared__ float As[SK][ST + 1];  // As[k][m]
  __shared__ float Bs[SK][ST + 1];  // Bs[k][n]
  if (gptq::status_bad(status)) return;
  const int m0 = blockIdx.y * ST, n0 = blockIdx.x * ST;
  if (upper_only && m0 > n0 + ST - 1) return;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  float acc[2][2] = {};
  int k_lo, k_hi;
  gptq_host::tri_k_range(tri, m0, n0, n0 + ST, K, k_lo, k_hi);
  for (int k0 = k_lo / SK * SK; k0 < k_hi; k0 += SK) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int e = tid + 256 * r;  // 1024 elements per operand slab
      int mm, kk;
      if (transA) { mm = e & 31; kk = e >> 5; } else { kk = e & 31; mm = e >> 5; }
      const int gm = m0 + mm, gk = k0 + kk;
      As[kk][mm] = (gm < M && gk < K) ? (transA ? A[(long long)gk * lda + gm] : A[(long long)gm * lda + gk]) : 0.f;
      int nn, kb;
      if (!transB) { nn = e & 31; kb = e >> 5; } else { kb = e & 31; nn = e >> 5; }
      const int gn = n0 + nn, gkb = k0 + kb;
      Bs[kb][nn] = (gn < N && gkb < K) ? (transB ? B[(long long)gn * ldb + gkb] : B[(long long)gkb * ldb + gn]) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < SK; ++kk) {
      const float a0 = As[kk][ty], a1 = As[kk][ty + 16];
      const float b0 = Bs[kk][tx], b1 = Bs[kk][tx + 16];
      acc[0][0] = fmaf(a0, b0, acc[0][0]);
      acc[0][1] = fmaf(a0, b1, acc[0][1]);
      acc[1][0] = fmaf(a1, b0, acc[1][0]);
      acc[1][1] = fmaf(a1, b1, acc[1][1]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int gm = m0 + ty + 16 * i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int gn = n0 + tx + 16 * j;
      if (gn >= N || (upper_only && gm > gn)) continue;
      float* cp = C + (long long)gm * ldc + gn;
      const float v = alpha * acc[i][j];
      *cp = (beta == 0.f) ? v : fmaf(beta, *cp, v);
    }
  }
}

// Staged GEMMs for short inner dimensions: one CTA per TM x 32 output tile (TM = 32 or 64),
// 256 threads. The tile's k-range (after the triangular restriction) is brought into shared
// memory in chunks: every thread issues all of its 16-byte loads of a chunk before storing any,
// so a chunk costs one memory round trip, and C (when beta != 0) is fetched together with the
// first chunk. Shared memory holds both operands k-major; an operand stored with k contiguous in
// memory is transposed on the way in, with consecutive lanes on consecutive rows so that the
// transposing stores hit distinct banks. The 8 warps form TM/32 groups, one per 32-row half;
// the warps of a group split the chunk's k-range over the whole 32 x 32 half (lane: 4 rows x 8
// columns, operands read as float4) and their partial sums are added through shared memory at
// the end. The 64-row tile halves the CTA count of tall products so that they run in one wave.
// Needs 16-byte aligned A and B, leading dimensions and K multiples of 4.
constexpr int G_THREADS = 256, GPB = 36;
template <int TM> struct Staged {
  static constexpr int KC = TM == 32 ? 256 : 128;       // chunk length
  static constexpr int PA = TM + 4;                     // row pitch of As[k][m]
  static constexpr int SMEM = KC * (PA + GPB) * 4;      // 72 KB / 52 KB
  static constexpr int PER_A = TM * KC / 4 / G_THREADS; // 16-byte granules per thread (8)
  static constexpr int PER_B = 32 * KC / 4 / G_THREADS; // 8 / 4
  static constexpr int GROUPS = TM / 32;
  static constexpr int WPG = 8 / GROUPS;                // warps per 32-row group
  static constexpr int OUT = TM * 32 / G_THREADS;       // outputs per thread in the epilogue
};

template <int TM>
__global__ void __launch_bounds__(G_THREADS)
gemm_f32_staged_kernel(int M, int N, int K, float alpha, const float* __restrict__ A,
                       long long lda, int transA, const float* __restrict__ B, long long ldb,
                       int transB, float beta, float* __restrict__ C, long long ldc,
                       int upper_only, int tri, const int32_t* status) {
  using P = Staged<TM>;
  extern __shared__ __align__(16) float gsm[];
  float* As = gsm;                   // As[k][m], k relative to the chunk start
  float* Bs = gsm + P::KC * P::PA;   // Bs[k][n]
  if (gptq::status_bad(status)) return;
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * 32;
  if (upper_only && m0 > n0 + 31) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = warp / P::WPG, kpart = warp % P::WPG;
  const int r4 = 32 * grp + 4 * (lane >> 2), c8 = 8 * (lane & 3);
  int k_lo, k_hi;
  gptq_host::tri_k_range(tri, m0, n0, n0 + 32, K, k_lo, k_hi);
  k_lo &= ~3;

  // C of this thread's epilogue outputs, fetched now so that its latency overlaps the operands'.
  float cpre[P::OUT];
#pragma unroll
  for (int q = 0; q < P::OUT; ++q) {
    const int e = tid + q * G_THREADS, gm = m0 + (e >> 5), gn = n0 + (e & 31);
    cpre[q] = (beta != 0.f && gm < M && gn < N && !(upper_only && gm > gn))
                  ? C[(long long)gm * ldc + gn] : 0.f;
  }

  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  for (int kc = k_lo; kc < k_hi; kc += P::KC) {
    const int kn = min(P::KC, k_hi - kc);  // a multiple of 4
    const int kq = kn >> 2;
    float4 va[P::PER_A], vb[P::PER_B];
    // op(A)[m0 + mm][kc + kk] and op(B)[kc + kk][n0 + nn]; granules run along the contiguous
    // direction of each operand in memory.
#pragma unroll
    for (int q = 0; q < P::PER_A; ++q) {
      const int g = tid + q * G_THREADS;
      va[q] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (g < TM * kq) {
        if (!transA) {  // A[m][k]: granule = 4 consecutive k of row mm (lanes along m)
          const int mm = g % TM, kk = 4 * (g / TM);
          if (m0 + mm < M)
            va[q] = *reinterpret_cast<const float4*>(A + (long long)(m0 + mm) * lda + kc + kk);
        } else {        // A[k][m]: granule = 4 consecutive m of row kk
          const int kk = g / (TM / 4), mm = 4 * (g % (TM / 4));
          const float* src = A + (long long)(kc + kk) * lda + m0 + mm;
          if (m0 + mm + 4 <= M) {
            va[q] = *reinterpret_cast<const float4*>(src);
          } else {
            if (m0 + mm + 0 < M) va[q].x = src[0];
            if (m0 + mm + 1 < M) va[q].y = src[1];
            if (m0 + mm + 2 < M) va[q].z = src[2];
          }
        }
      }
    }
#pragma unroll
    for (int q = 0; q < P::PER_B; ++q) {
      const int g = tid + q * G_THREADS;
      vb[q] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (g < 32 * kq) {
        if (transB) {   // B[n][k]: granule = 4 consecutive k of row nn (lanes along n)
          const int nn = g & 31, kk = 4 * (g >> 5);
          if (n0 + nn < N)
            vb[q] = *reinterpret_cast<const float4*>(B + (long long)(n0 + nn) * ldb + kc + kk);
        } else {        // B[k][n]: granule = 4 consecutive n of row kk
          const int kk = g >> 3, nn = 4 * (g & 7);
          const float* src = B + (long long)(kc + kk) * ldb + n0 + nn;
          if (n0 + nn + 4 <= N) {
            vb[q] = *reinterpret_cast<const float4*>(src);
          } else {
            if (n0 + nn + 0 < N) vb[q].x = src[0];
            if (n0 + nn + 1 < N) vb[q].y = src[1];
            if (n0 + nn + 2 < N) vb[q].z = src[2];
          }
        }
      }
    }
#pragma unroll
    for (int q = 0; q < P::PER_A; ++q) {
      const int g = tid + q * G_THREADS;
      if (g < TM * kq) {
        if (!transA) {
          const int mm = g % TM, kk = 4 * (g / TM);
          As[(kk + 0) * P::PA + mm] = va[q].x;
          As[(kk + 1) * P::PA + mm] = va[q].y;
          As[(kk + 2) * P::PA + mm] = va[q].z;
          As[(kk + 3) * P::PA + mm] = va[q].w;
        } else {
          *reinterpret_cast<float4*>(As + (g / (TM / 4)) * P::PA + 4 * (g % (TM / 4))) = va[q];
        }
      }
    }
#pragma unroll
    for (int q = 0; q < P::PER_B; ++q) {
      const int g = tid + q * G_THREADS;
      if (g < 32 * kq) {
        if (transB) {
          const int nn = g & 31, kk = 4 * (g >> 5);
          Bs[(kk + 0) * GPB + nn] = vb[q].x;
          Bs[(kk + 1) * GPB + nn] = vb[q].y;
          Bs[(kk + 2) * GPB + nn] = vb[q].z;
          Bs[(kk + 3) * GPB + nn] = vb[q].w;
        } else {
          *reinterpret_cast<float4*>(Bs + (g >> 3) * GPB + 4 * (g & 7)) = vb[q];
        }
      }
    }
    __syncthreads();
    const int kw = (kn + P::WPG - 1) / P::WPG;
    const int kb = kpart * kw, ke = min(kn, kb + kw);
#pragma unroll 4
    for (int k = kb; k < ke; ++k) {
      const float4 a = *reinterpret_cast<const float4*>(As + k * P::PA + r4);
      const float4 b0 = *reinterpret_cast<const float4*>(Bs + k * GPB + c8);
      const float4 b1 = *reinterpret_cast<const float4*>(Bs + k * GPB + c8 + 4);
      const float av[4] = {a.x, a.y, a.z, a.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();  // the next chunk (or the reduction) overwrites the staging area
  }
  // Partial sums of the warps -> shared memory (8 x 32 x 33 floats, inside the staging area),
  // then each thread finishes OUT outputs by adding its group's WPG partials.
  float* red = gsm;
  const int rl = 4 * (lane >> 2);
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) red[(warp * 32 + rl + i) * 33 + c8 + j] = acc[i][j];
  __syncthreads();
#pragma unroll
  for (int q = 0; q < P::OUT; ++q) {
    const int e = tid + q * G_THREADS, row = e >> 5, col = e & 31;
    const int g = row >> 5, r = row & 31;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < P::WPG; ++w) v += red[((g * P::WPG + w) * 32 + r) * 33 + col];
    const int gm = m0 + row, gn = n0 + col;
    if (gm >= M || gn >= N || (upper_only && gm > gn)) continue;
    v *= alpha;
    C[(long long)gm * ldc + gn] = (beta == 0.f) ? v : fmaf(beta, cpre[q], v);
  }
}

}  // namespace

namespace gptq_host {

int gemm_f32_small(int M, int N, int K, float alpha, const float* A, long long lda, bool transA,
                   const float* B, long long ldb, bool transB, float beta, float* C,
                   long long ldc, bool upper_only, const int32_t* status, cudaStream_t stream,
                   int tri) {
  dim3 grid((N + ST - 1) / ST, (M + ST - 1) / ST);
  gemm_f32_small_kernel<<<grid, 256, 0, stream>>>(M, N, K, alpha, A, lda, transA ? 1 : 0, B, ldb,
                                                  transB ? 1 : 0, beta, C, ldc,
                                                  upper_only ? 1 : 0, tri, status);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

bool gemm_f32_staged_supported(int K, const float* A, long long lda, const float* B,
                               long long ldb) {
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  return K > 0 && (K % 4) == 0 && al16(A) && al16(B) && (lda % 4) == 0 && (ldb % 4) == 0;
}

int gemm_f32_staged(int M, int N, int K, float alpha, const float* A, long long lda, bool transA,
                    const float* B, long long ldb, bool transB, float beta, float* C,
                    long long ldc, bool upper_only, const int32_t* status, cudaStream_t stream,
                    int tri, bool exclusive) {
  if (M <= 0 || N <= 0) return 0;
  constexpr int kExclusiveSmem = 160 * 1024;  // > 227 KB - 72 KB: nothing else fits beside it
  // 64-row tiles when 32-row ones would need more than one wave (two CTAs per SM).
  const long long tiles32 = (long long)((N + 31) / 32) * ((M + 31) / 32);
  if (tiles32 > 2LL * num_sms() && M >= 64) {
    const int smem = exclusive ? kExclusiveSmem : Staged<64>::SMEM;
    if (ensure_smem_attr(reinterpret_cast<const void*>(gemm_f32_staged_kernel<64>), smem) != 0)
      return GPTQ_ERR_CUDA;
    dim3 grid((N + 31) / 32, (M + 63) / 64);
    gemm_f32_staged_kernel<64><<<grid, G_THREADS, smem, stream>>>(
        M, N, K, alpha, A, lda, transA ? 1 : 0, B, ldb, transB ? 1 : 0, beta, C, ldc,
        upper_only ? 1 : 0, tri, status);
  } else {
    const int smem = exclusive ? kExclusiveSmem : Staged<32>::SMEM;
    if (ensure_smem_attr(reinterpret_cast<const void*>(gemm_f32_staged_kernel<32>), smem) != 0)
      return GPTQ_ERR_CUDA;
    dim3 grid((N + 31) / 32, (M + 31) / 32);
    gemm_f32_staged_kernel<32><<<grid, G_THREADS, smem, stream>>>(
        M, N, K, alpha, A, lda, transA ? 1 : 0, B, ldb, transB ? 1 : 0, beta, C, ldc,
        upper_only ? 1 : 0, tri, status);
  }
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

// CUDA-core GEMM: used only where TMA cannot address the operands (row strides or bases not
// 16-byte aligned) and for K = 0; everything else goes to the tcgen05 3xTF32 kernel.
int gemm_f32_simt(int M, int N, int K, float alpha, const float* A, long long lda, bool transA,
                  const float* B, long long ldb, bool transB, float beta, float* C, long long ldc,
                  bool upper_only, const int32_t* status, cudaStream_t stream, int tri) {
  if (M <= 0 || N <= 0) return 0;
  dim3 grid((N + TN - 1) / TN, (M + TM - 1) / TM);
  gemm_f32_simt_kernel<<<grid, THREADS, 0, stream>>>(M, N, K, alpha, A, lda, transA ? 1 : 0, B,
                                                     ldb, transB ? 1 : 0, beta, C, ldc,
                                                     upper_only ? 1 : 0, tri, status);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

}  // namespace gptq_host

namespace gptq_host {

int gemm_f32(int M, int N, int K, float alpha, const float* A, long long lda, bool transA,
             const float* B, long long ldb, bool transB, float beta, float* C, long long ldc,
             bool upper_only, const int32_t* status, cudaStream_t stream, int tri,
             int max_ctas, bool exclusive) {
  if (M <= 0 || N <= 0) return 0;
  // Products up to 512 x 512 x 512 (the lower levels of the U recursion) finish sooner on
  // 32 x 32 CUDA-core tiles with the k-range staged in one round than through the tensor-core
  // pipeline's fill latency (graph replay: 128^3 4.7 us vs 12.3 us, 256^3 6.4 vs 15.8, 512^3
  // 16.3 vs 22.4); larger ones go to tcgen05 (3xTF32).
  if (K <= 512 && (long long)M * N <= 512LL * 512 && gemm_f32_staged_supported(K, A, lda, B, ldb))
    return gemm_f32_staged(M, N, K, alpha, A, lda, transA, B, ldb, transB, beta, C, ldc,
                           upper_only, status, stream, tri, exclusive);
  if ((long long)M * N <= 4LL * 128 * 128)
    return gemm_f32_small(M, N, K, alpha, A, lda, transA, B, ldb, transB, beta, C, ldc,
                          upper_only, status, stream, tri);
  if (gemm_tf32x3_supported(M, N, K, A, lda, B, ldb, C, ldc))
    return gemm_tf32x3(M, N, K, alpha, A, lda, transA, B, ldb, transB, beta, C, ldc, upper_only,
                       status, stream, tri, max_ctas);
  return gemm_f32_simt(M, N, K, alpha, A, lda, transA, B, ldb, transB, beta, C, ldc, upper_only,
                       status, stream, tri);
}

}  // namespace gptq_host
