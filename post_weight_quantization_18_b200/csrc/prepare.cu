// prepare.cu — numerical preparation of the Hessian on the GPU.
//
// "GPTQ: Mathematical Foundations ...":
//   §Activation Ordering (Act-Order / Desc-Act): pi = argsort(diag(H), descending),
//     H <- H[pi][:, pi] (stable order: equal keys keep the lower index first).
//   §GPTQ Algorithm Execution Walkthrough, step 1: dead columns (diag 0) get H_jj = 1; the
//     damping lambda = percdamp * mean(diag H) is added to the diagonal
//     (§Hessian Damping and Numerical Regularization).
//   §3 Cholesky Decomposition and Pre-computation: U upper with H^-1 = U^T U.
//
// U is obtained without forming H^-1: factor H_d = V V^T with V upper triangular (Cholesky
// from the last column), then U = V^-1. (V^-T V^-1 = H_d^-1 and V^-1 is upper with a positive
// diagonal, so it is the unique upper Cholesky factor of H_d^-1.) The host schedule in api.cu
// runs right-looking over 128-column blocks up to 4096 columns (splitting larger matrices in
// halves first) and does the off-diagonal work with GEMMs; each 128-column diagonal block is
// factored and inverted here by one CTA in shared memory.
#include "common.cuh"
#include "kernels.h"
#include "tri_fill.cuh"

namespace {

// Hp[a][b] = H[pi a][pi b] on the upper triangle, reading H's upper triangle symmetrically:
// rows on grid y, columns of the row's span strided over grid x (tri_fill.cuh).
__global__ void permute_sym_kernel(const float* __restrict__ H, float* __restrict__ Hp,
                                   const int32_t* __restrict__ perm, int d,
                                   const int32_t* status) {
  if (gptq::status_bad(status)) return;
  for (long long a = blockIdx.y; a < d; a += gridDim.y) {
    long long lo, hi;
    gptq::tri_row_span(gptq::kUpperWithDiag, a, d, lo, hi);
    const int pa = perm[a];
    for (long long b = lo + blockIdx.x * (long long)blockDim.x + threadIdx.x; b < hi;
         b += (long long)gridDim.x * blockDim.x)
      gptq::permute_sym_elem(H, Hp, perm, d, a, pa, b);
  }
}

// dst's upper triangle (with the diagonal) = src's, same layout.
__global__ void copy_upper_kernel(const float* __restrict__ src, float* __restrict__ dst, int d,
                                  const int32_t* status) {
  if (gptq::status_bad(status)) return;
  for (long long a = blockIdx.y; a < d; a += gridDim.y) {
    long long lo, hi;
    gptq::tri_row_span(gptq::kUpperWithDiag, a, d, lo, hi);
    for (long long b = lo + blockIdx.x * (long long)blockDim.x + threadIdx.x; b < hi;
         b += (long long)gridDim.x * blockDim.x)
      dst[a * d + b] = src[a * d + b];
  }
}

// Stable descending rank of diag(H): rank_i = #{j : h_j > h_i or (h_j == h_i and j < i)};
// perm[rank_i] = i.
__global__ void act_order_rank_kernel(const float* __restrict__ H, int32_t* __restrict__ perm,
                                      int d, const int32_t* status) {
  __shared__ float keys[1024];
  __shared__ int bad;  // read once per block: every thread takes the same branch
  if (threadIdx.x == 0) bad = gptq::status_bad(status) ? 1 : 0;
  __syncthreads();
  if (bad) return;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const float hi = (i < d) ? H[(long long)i * d + i] : 0.f;
  int rank = 0;
  for (int base = 0; base < d; base += 1024) {
    for (int t = threadIdx.x; t < 1024; t += blockDim.x) {
      const int j = base + t;
      keys[t] = (j < d) ? H[(long long)j * d + j] : 0.f;
    }
    __syncthreads();
    const int lim = min(1024, d - base);
    if (i < d) {
      for (int t = 0; t < lim; ++t) {
        const float hj = keys[t];
        const int j = base + t;
        rank += (hj > hi || (hj == hi && j < i)) ? 1 : 0;
      }
    }
    __syncthreads();
  }
  if (i < d) perm[rank] = i;
}

__global__ void identity_perm_kernel(int32_t* perm, int d, const int32_t* status) {
  if (gptq::status_bad(status)) return;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < d; i += gridDim.x * blockDim.x)
    perm[i] = i;
}

// One CTA: dead-column fix, mean of the diagonal (after the fix), damping.
__global__ void dead_damp_kernel(float* __restrict__ H, uint8_t* __restrict__ dead, int d,
                                 float percdamp, int32_t* status) {
  __shared__ double partial[32];
  __shared__ int bad;
  __shared__ float lam_s;
  if (threadIdx.x == 0) bad = gptq::status_bad(status) ? 1 : 0;
  __syncthreads();
  if (bad) return;
  double acc = 0.0;
  int nonfinite = -1;
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    float h = H[(long long)j * d + j];
    if (!isfinite(h)) nonfinite = j;
    const bool is_dead = (h == 0.0f);
    dead[j] = is_dead ? 1 : 0;
    if (is_dead) {
      h = 1.0f;
      H[(long long)j * d + j] = 1.0f;
    }
    acc += (double)h;
  }
  if (nonfinite >= 0) gptq::set_status(status, GPTQ_ERR_NONFINITE, nonfinite);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) partial[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += partial[w];
    lam_s = (float)((double)percdamp * (s / (double)d));
  }
  __syncthreads();
  const float lam = lam_s;
  for (int j = threadIdx.x; j < d; j += blockDim.x) H[(long long)j * d + j] += lam;
}

// U's strictly lower triangle = 0: rows over the blocks, 16-byte stores along each row's span
// (tri_fill.cuh).
__global__ void zero_lower_kernel(float* U, int d, const int32_t* status) {
  if (gptq::status_bad(status)) return;
  for (long long r = blockIdx.x; r < d; r += gridDim.x) {
    long long lo, hi;
    gptq::tri_row_span(gptq::kStrictLower, r, d, lo, hi);
    gptq::fill_span(U + r * d, lo, hi, 0.f, threadIdx.x, blockDim.x);
  }
}

// Base block (n <= 128): the damped block H_d (upper triangle, leading dimension ld) -> the
// U block = V^-1 where H_d = V V^T, V upper. A recursion on halves (the one the host uses above
// 4096 columns), inside one CTA of 16 warps on two shared-memory matrices (A: the block being
// factored, U: the result): 128 -> 64 -> 32 -> 16-column leaves. Each split does its four
// block products on the tensor cores (warp-level m16n8k8 TF32 with the three-term hi/lo split,
// so the products carry fp32 accuracy), skipping the k-ranges where the triangular operand is
// zero and computing only the upper tiles of the symmetric update. A 32-column node (two
// leaves and its four 16 x 16 products) runs on one warp without block barriers; a leaf is
// factored and inverted in registers.
// A block smaller than 128 is padded at its end with the identity: the padded factor is block
// diagonal, so the leading n x n part is unchanged.
constexpr int BASE_THREADS = 512;
constexpr int BASE_WARPS = BASE_THREADS / 32;
constexpr int BN_ = gptq_host::kPrepBase;  // 128
// Row pitch of the shared-memory matrices. 132 = 4 (mod 32) puts rows g = 0..7 of a fragment
// on banks 4g, so the 8 rows x 4 columns that an m16n8k8 operand fragment reads hit 32
// distinct banks; rows stay 16-byte aligned for vector copies.
constexpr int BLD = BN_ + 4;
constexpr int U_OFF = BN_ * BLD;           // U follows A in shared memory
constexpr int kLeaf = 16;

// Leaf: A[o:o+16, o:o+16] (upper part) -> U[o:o+16, o:o+16] (upper, zeros below). One warp.
//   Cholesky from the last column, lane r owning row r: at step j the pivot a_jj arrives by
//   shuffle, V_rj = a_rj / sqrt(a_jj) is formed by each lane for its own row and kept in
//   registers (vrow), and a_rk -= V_rj V_kj for r <= k < j with V_kj shuffled from lane k.
//   Inverse by back substitution with lane c owning column c of U (U V = I read column-wise:
//   V U = I): U_cc = 1/V_cc = rsqrt(a_cc) and, for r < c, U_rc = -(sum_{r<k<=c} V_rk U_kc)/V_rr
//   with V_rk shuffled from lane r; the newest term enters each sum last.
// Returns -1, or the first leaf column (in factorization order) whose pivot is not positive
// and finite; the value is the same on every lane.
__device__ __noinline__ int leaf16(int o) {
  extern __shared__ float sm[];
  const int lane = threadIdx.x & 31;
  constexpr int N = kLeaf;
  float a[N], vrow[N], rinv[N];
#pragma unroll
  for (int c = 0; c < N; ++c) a[c] = (lane < N && c >= lane) ? sm[(o + lane) * BLD + o + c] : 0.f;
  int badj = -1;
  // dn: on lane j, the pivot of step j. The owner of the next pivot updates it from its own v,
  // so the next step waits for one FMA rather than for this step's shuffles (same value as the
  // shuffled update of a[j - 1] below).
  float dn = a[N - 1];
#pragma unroll
  for (int j = N - 1; j >= 0; --j) {
    const float piv = __shfl_sync(0xffffffffu, dn, j);
    if (badj < 0 && !(piv > 0.f && piv <= 3.402823466e38f)) badj = j;
    // Reciprocal square root from the special-function unit (about 1 ulp, the order of the
    // factor's own fp32 rounding).
    const float inv = rsqrtf(piv);
    rinv[j] = inv;
    const float v = (lane < j) ? a[j] * inv : (lane == j ? piv * inv : 0.f);
    vrow[j] = v;
    if (j > 0) dn = fmaf(-v, v, a[j - 1]);
#pragma unroll
    for (int k = 0; k < j; ++k) {
      const float vk = __shfl_sync(0xffffffffu, v, k);
      if (k >= lane) a[k] = fmaf(-v, vk, a[k]);
    }
  }
  float u[N];
#pragma unroll
  for (int r = N - 1; r >= 0; --r) {
    float s = 0.f;
#pragma unroll
    for (int k = N - 1; k > r; --k) s = fmaf(__shfl_sync(0xffffffffu, vrow[k], r), u[k], s);
    u[r] = (r == lane) ? rinv[r] : (r < lane ? -s * rinv[r] : 0.f);
  }
  if (lane < N) {
#pragma unroll
    for (int k = 0; k < N; ++k) sm[U_OFF + (o + k) * BLD + o + lane] = u[k];
  }
  __syncwarp();
  return badj;
}

// Which operand of a block product is triangular, so that whole k-steps can be skipped, or
// whether only the upper output tiles are wanted.
enum : int {
  kFull = 0,
  kYUpperTransposed = 1,  // Y[n][k] upper (read transposed): terms with k < n vanish
  kCUpperOnly = 2,        // symmetric result: output tiles below the diagonal are not needed
  kYUpper = 3,            // Y[k][n] upper: terms with k > n vanish
  kXUpper = 4,            // X[i][k] upper: terms with k < i vanish
};

GPTQ_DEV uint32_t tf32_hi(float x) { return __float_as_uint(x) & 0xffffe000u; }
GPTQ_DEV uint32_t tf32_lo(float x, uint32_t hi) { return __float_as_uint(x - __uint_as_float(hi)); }

GPTQ_DEV void mma_m16n8k8_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// C (M x M) = alpha * X Y' + beta * C on shared-memory blocks (offsets into the dynamic shared
// array, pitch BLD), Y' = Y^T (Y read as Y[n][k]) for the transposed kinds and Y (Y[k][n])
// otherwise. Warps w0 .. w0+nw-1 take 16 x 16 output tiles in turn. Each product x*y is formed
// as hi(x)hi(y) + hi(x)lo(y) + lo(x)hi(y) with hi the operand's top 19 bits (TF32) and lo the
// rest. One instance per (M, TRI), so that the k-loop is unrolled and the operand layout fixed
// at compile time.
template <int M, int TRI>
__device__ __noinline__ void block_mma(int c_off, int x_off, int y_off, float alpha, float beta,
                                       int w0, int nw) {
  extern __shared__ float sm[];
  constexpr bool kYT = (TRI == kYUpperTransposed || TRI == kCUpperOnly);
  constexpr int kTiles = M / 16;
  const int warp = (threadIdx.x >> 5) - w0, lane = threadIdx.x & 31;
  if (warp < 0 || warp >= nw) return;
  const int g = lane >> 2, t = lane & 3;
  const float* X = sm + x_off;
  const float* Y = sm + y_off;
  float* C = sm + c_off;
  for (int tile = warp; tile < kTiles * kTiles; tile += nw) {
    const int i0 = (tile / kTiles) * 16, n0 = (tile % kTiles) * 16;
    if (TRI == kCUpperOnly && i0 > n0) continue;
    int k_lo = 0, k_hi = M;
    if (TRI == kYUpperTransposed) k_lo = n0;
    if (TRI == kYUpper) k_hi = n0 + 16;
    if (TRI == kXUpper) k_lo = i0;
    float hh[2][4] = {}, cross[2][4] = {};
#pragma unroll
    for (int k0 = 0; k0 < M; k0 += 8) {
      if (k0 < k_lo || k0 >= k_hi) continue;
      const float xa[4] = {X[(i0 + g) * BLD + k0 + t], X[(i0 + g + 8) * BLD + k0 + t],
                           X[(i0 + g) * BLD + k0 + t + 4], X[(i0 + g + 8) * BLD + k0 + t + 4]};
      uint32_t ah[4], al[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        ah[q] = tf32_hi(xa[q]);
        al[q] = tf32_lo(xa[q], ah[q]);
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int n = n0 + 8 * h + g;
        const float y0 = kYT ? Y[n * BLD + k0 + t] : Y[(k0 + t) * BLD + n];
        const float y1 = kYT ? Y[n * BLD + k0 + t + 4] : Y[(k0 + t + 4) * BLD + n];
        const uint32_t bh0 = tf32_hi(y0), bh1 = tf32_hi(y1);
        mma_m16n8k8_tf32(cross[h], ah, tf32_lo(y0, bh0), tf32_lo(y1, bh1));
        mma_m16n8k8_tf32(cross[h], al, bh0, bh1);
        mma_m16n8k8_tf32(hh[h], ah, bh0, bh1);
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float* cp = C + (i0 + g + ((q & 2) ? 8 : 0)) * BLD + n0 + 8 * h + 2 * t + (q & 1);
        const float v = alpha * (hh[h][q] + cross[h][q]);
        *cp = (beta == 0.f) ? v : fmaf(beta, *cp, v);
      }
  }
}

// Offsets of the blocks of one split: node [o, o+N) split at m = N/2.
struct Split {
  int Bb, Aa, U11, U12, U22;
  __device__ Split(int o, int m)
      : Bb(o * BLD + o + m),                 // A[o:o+m, o+m:o+N]
        Aa(o * BLD + o),                     // A[o:o+m, o:o+m]
        U11(U_OFF + o * BLD + o),
        U12(U_OFF + o * BLD + o + m),
        U22(U_OFF + (o + m) * BLD + o + m) {}
};

// A 32-column node [o, o+32) entirely on warp 0: two 16-column leaves and the four 16 x 16
// products of the split, ordered by __syncwarp only. Returns -1 or the failing column (within
// the node) of the first non-positive pivot; the value is the same on every lane of warp 0.
__device__ __forceinline__ int node32_warp(int o) {
  const Split sp(o, 16);
  int bad = leaf16(o + 16);
  if (bad >= 0) return 16 + bad;
  block_mma<16, kYUpperTransposed>(sp.U12, sp.Bb, sp.U22, 1.f, 0.f, 0, 1);  // T = B U22^T
  __syncwarp();
  block_mma<16, kCUpperOnly>(sp.Aa, sp.U12, sp.U12, -1.f, 1.f, 0, 1);      // S = A - T T^T
  block_mma<16, kYUpper>(sp.Bb, sp.U12, sp.U22, 1.f, 0.f, 0, 1);           // V = T U22
  __syncwarp();
  bad = leaf16(o);
  if (bad >= 0) return bad;
  block_mma<16, kXUpper>(sp.U12, sp.U11, sp.Bb, -1.f, 0.f, 0, 1);          // U12 = -U11 V
  __syncwarp();
  return -1;
}

template <int N>
__device__ __forceinline__ bool base_rec(int o, int32_t* status, int index0, int* fail) {
  if constexpr (N == 32) {
    if (threadIdx.x < 32) {
      const int bad = node32_warp(o);
      if (bad >= 0 && threadIdx.x == 0) {
        gptq::set_status(status, GPTQ_ERR_NOT_SPD, index0 + o + bad);
        *fail = 1;
      }
    }
    __syncthreads();
    return *fail == 0;
  } else {
    constexpr int m = N / 2;
    const Split sp(o, m);
    if (!base_rec<m>(o + m, status, index0, fail)) return false;
    block_mma<m, kYUpperTransposed>(sp.U12, sp.Bb, sp.U22, 1.f, 0.f, 0, BASE_WARPS);  // T
    __syncthreads();
    // S = A - T T^T (upper tiles) and V = T U22 both need only T: one barrier for the two.
    block_mma<m, kCUpperOnly>(sp.Aa, sp.U12, sp.U12, -1.f, 1.f, 0, BASE_WARPS / 2);
    block_mma<m, kYUpper>(sp.Bb, sp.U12, sp.U22, 1.f, 0.f, BASE_WARPS / 2, BASE_WARPS / 2);
    __syncthreads();
    if (!base_rec<m>(o, status, index0, fail)) return false;
    block_mma<m, kXUpper>(sp.U12, sp.U11, sp.Bb, -1.f, 0.f, 0, BASE_WARPS);        // U12
    __syncthreads();
    return true;
  }
}

__global__ void __launch_bounds__(BASE_THREADS, 1)
base_block_kernel(const float* __restrict__ Hblk, float* __restrict__ Ublk, int n, int ld,
                  int index0, int32_t* status) {
  extern __shared__ float sm[];
  __shared__ int bad, fail;
  if (threadIdx.x == 0) {
    bad = gptq::status_bad(status) ? 1 : 0;
    fail = 0;
  }
  const bool vec = (n == BN_) && (ld % 4 == 0) && ((reinterpret_cast<uintptr_t>(Hblk) & 15) == 0) &&
                   ((reinterpret_cast<uintptr_t>(Ublk) & 15) == 0);
  if (vec) {
    // Full block: all eight 16-byte loads of a thread are issued before any is used.
    constexpr int kPer = BN_ * BN_ / 4 / BASE_THREADS;  // 8
    float4 v[kPer];
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int e = (q * BASE_THREADS + threadIdx.x) * 4, i = e / BN_, k = e % BN_;
      v[q] = *reinterpret_cast<const float4*>(Hblk + (long long)i * ld + k);
    }
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int e = (q * BASE_THREADS + threadIdx.x) * 4, i = e / BN_, k = e % BN_;
      *reinterpret_cast<float4*>(sm + i * BLD + k) = v[q];
      *reinterpret_cast<float4*>(sm + U_OFF + i * BLD + k) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  } else {
    for (int e = threadIdx.x; e < BN_ * BN_; e += BASE_THREADS) {
      const int i = e / BN_, k = e % BN_;
      float v = 0.f;
      if (i < n && k < n) v = (i <= k) ? Hblk[(long long)i * ld + k] : 0.f;
      else if (i == k) v = 1.f;  // identity padding at the end
      sm[i * BLD + k] = v;
      sm[U_OFF + i * BLD + k] = 0.f;
    }
  }
  __syncthreads();
  if (bad) return;
  if (!base_rec<BN_>(0, status, index0, &fail)) return;
  if (vec) {
    constexpr int kPer = BN_ * BN_ / 4 / BASE_THREADS;
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int e = (q * BASE_THREADS + threadIdx.x) * 4, i = e / BN_, k = e % BN_;
      float4 v = *reinterpret_cast<const float4*>(sm + U_OFF + i * BLD + k);
      // The shared U is zero below the diagonal already; the mask makes the output's lower
      // triangle independent of that.
      if (k + 0 < i) v.x = 0.f;
      if (k + 1 < i) v.y = 0.f;
      if (k + 2 < i) v.z = 0.f;
      if (k + 3 < i) v.w = 0.f;
      *reinterpret_cast<float4*>(Ublk + (long long)i * ld + k) = v;
    }
  } else {
    for (int e = threadIdx.x; e < n * n; e += BASE_THREADS) {
      const int i = e / n, k = e % n;
      Ublk[(long long)i * ld + k] = (i <= k) ? sm[U_OFF + i * BLD + k] : 0.f;
    }
  }
}

inline int grid_for(long long total) {
  long long g = (total + 255) / 256;
  const long long cap = (long long)gptq_host::num_sms() * 8;
  return (int)(g < 1 ? 1 : (g > cap ? cap : g));
}

}  // namespace

namespace gptq_host {

int prep_permute_sym(const float* H, float* Hp, const int32_t* perm, int d,
                     const int32_t* status, cudaStream_t stream) {
  const dim3 grid((unsigned)((d + 1023) / 1024), (unsigned)(d < 65535 ? d : 65535));
  permute_sym_kernel<<<grid, 256, 0, stream>>>(H, Hp, perm, d, status);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int prep_copy_upper(const float* src, float* dst, int d, const int32_t* status,
                    cudaStream_t stream) {
  const dim3 grid((unsigned)((d + 1023) / 1024), (unsigned)(d < 65535 ? d : 65535));
  copy_upper_kernel<<<grid, 256, 0, stream>>>(src, dst, d, status);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int prep_act_order(const float* H, int32_t* perm, int d, const int32_t* status,
                   cudaStream_t stream) {
  act_order_rank_kernel<<<(d + 255) / 256, 256, 0, stream>>>(H, perm, d, status);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int prep_identity_perm(int32_t* perm, int d, const int32_t* status, cudaStream_t stream) {
  identity_perm_kernel<<<grid_for(d), 256, 0, stream>>>(perm, d, status);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int prep_dead_damp(float* H, uint8_t* dead, int d, float percdamp, int32_t* status,
                   cudaStream_t stream) {
  dead_damp_kernel<<<1, 1024, 0, stream>>>(H, dead, d, percdamp, status);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int prep_zero_lower(float* U, int d, const int32_t* status, cudaStream_t stream) {
  const int grid = d < num_sms() * 8 ? d : num_sms() * 8;
  zero_lower_kernel<<<grid, 256, 0, stream>>>(U, d, status);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int prep_base_block(float* Hblk, float* Ublk, int n, int ld, int index0, int32_t* status,
                    cudaStream_t stream) {
  // The block uses 2 * 128 * 132 floats of shared memory; it asks for 180 KB so that no CTA of
  // the products running beside it on other streams (up to 72 KB) shares its SM: the block is
  // a single latency-bound CTA on the critical path and runs at its own speed only alone.
  const size_t smem_used = 2 * (size_t)kPrepBase * BLD * sizeof(float);
  const size_t smem = smem_used > 180 * 1024 ? smem_used : 180 * 1024;
  if (ensure_smem_attr(reinterpret_cast<const void*>(base_block_kernel), (int)smem) != 0)
    return GPTQ_ERR_CUDA;
  base_block_kernel<<<1, BASE_THREADS, smem, stream>>>(Hblk, Ublk, n, ld, index0, status);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

}  // namespace gptq_host
