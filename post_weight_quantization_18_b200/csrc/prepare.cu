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
// diagonal, so it is the unique upper Cholesky factor of H_d^-1.) The host recursion in
// api.cu splits the matrix into halves and uses GEMMs; the base blocks of at most 128 columns
// are factored and inverted here by one CTA in shared memory.
#include "common.cuh"
#include "kernels.h"

namespace {

// Hp[a][b] = H[pi a][pi b] on the upper triangle, reading H's upper triangle symmetrically.
__global__ void permute_sym_kernel(const float* __restrict__ H, float* __restrict__ Hp,
                                   const int32_t* __restrict__ perm, int d) {
  const long long total = (long long)d * d;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int a = (int)(e / d), b = (int)(e % d);
    if (a > b) continue;
    const int i = perm[a], j = perm[b];
    const int lo = i < j ? i : j, hi = i < j ? j : i;
    Hp[(long long)a * d + b] = H[(long long)lo * d + hi];
  }
}

__global__ void copy_upper_kernel(const float* __restrict__ src, float* __restrict__ dst, int d) {
  const long long total = (long long)d * d;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int a = (int)(e / d), b = (int)(e % d);
    if (a <= b) dst[e] = src[e];
  }
}

// Stable descending rank of diag(H): rank_i = #{j : h_j > h_i or (h_j == h_i and j < i)};
// perm[rank_i] = i.
__global__ void act_order_rank_kernel(const float* __restrict__ H, int32_t* __restrict__ perm,
                                      int d) {
  __shared__ float keys[1024];
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

__global__ void identity_perm_kernel(int32_t* perm, int d) {
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

__global__ void zero_lower_kernel(float* U, int d) {
  const long long total = (long long)d * d;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int a = (int)(e / d), b = (int)(e % d);
    if (a > b) U[e] = 0.f;
  }
}

// Base block (n <= 128): the damped block H_d (upper triangle, leading dimension ld) -> the
// U block = V^-1 where H_d = V V^T, V upper. The same recursion as the host one, inside one CTA:
//   128 -> 64 -> 32 on shared-memory matrices, with the four block products of every split
//   done by all 16 warps, and 32 x 32 leaves factored and inverted by a single warp entirely in
//   registers (lane = column; shuffles broadcast the pivot column, no block barriers).
// A block smaller than 128 is padded at its end with the identity: the padded factor is block
// diagonal, so the leading n x n part is unchanged.
constexpr int BASE_THREADS = 512;
constexpr int BN_ = gptq_host::kPrepBase;  // 128
constexpr int BLD = BN_ + 1;               // padded leading dimension (conflict-free columns)

// Leaf: A[o:o+32, o:o+32] (upper part) -> U[o:o+32, o:o+32] (upper, zeros below); one warp,
// lane r owns row r of the block in registers.
//   Cholesky from the last column: at step s the pivot column j = 31 - s sits in a[31] (the
//   registers rotate by one after every step, so the loop stays rolled with constant register
//   indices). V_rj = a_rj / sqrt(a_jj) is computed by each lane for its own row and kept in the
//   shared array V; then a_rk -= V_rj V_kj for r <= k < j with V_kj shuffled from lane k (the
//   31 shuffles of a step are independent of each other).
//   Inverse, row by row from U V = I: U_rc = (delta_rc - sum_{r<=k<c} U_rk V_kc) / V_cc, V read
//   from shared memory (one broadcast per element).
// Returns false (uniformly over the warp) on a non-positive or non-finite pivot.
constexpr int VLD = 33;

// One warp; N (16 or 32) rows, lanes >= N idle but present for the shuffles.
template <int N>
__device__ bool leaf(float* A, float* U, float* V, int o, int lane, int32_t* status,
                     int index0) {
  float a[N];
#pragma unroll
  for (int c = 0; c < N; ++c) a[c] = (lane < N && c >= lane) ? A[(o + lane) * BLD + o + c] : 0.f;
#pragma unroll 1
  for (int s = 0; s < N; ++s) {
    const int j = N - 1 - s;
    const float piv = __shfl_sync(0xffffffffu, a[N - 1], j);
    if (!(piv > 0.f) || !isfinite(piv)) {
      if (lane == 0) gptq::set_status(status, GPTQ_ERR_NOT_SPD, index0 + o + j);
      return false;
    }
    // Reciprocal square root from the special-function unit (about 1 ulp, the order of the
    // factor's own fp32 rounding).
    const float inv = rsqrtf(piv);
    const float v = (lane < j) ? a[N - 1] * inv : (lane == j ? piv * inv : 0.f);
    if (lane < N) V[lane * VLD + j] = v;
#pragma unroll
    for (int idx = 0; idx < N - 1; ++idx) {
      const int k = idx - s;  // column held in a[idx]
      const float vk = __shfl_sync(0xffffffffu, v, k & 31);
      if (k >= lane) a[idx] = fmaf(-v, vk, a[idx]);
    }
#pragma unroll
    for (int idx = N - 2; idx >= 0; --idx) a[idx + 1] = a[idx];
  }
  __syncwarp();
  if (lane < N) {
    float u[N];
#pragma unroll
    for (int c = 0; c < N; ++c) {
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int k = 0; k < c; ++k) {
        const float t = u[k] * V[k * VLD + c];
        if (k & 1) s1 += t;
        else s0 += t;
      }
      const float rc = __frcp_rn(V[c * VLD + c]);
      u[c] = (c == lane) ? rc : (c > lane ? -(s0 + s1) * rc : 0.f);
    }
#pragma unroll
    for (int c = 0; c < N; ++c) U[(o + lane) * BLD + o + c] = u[c];
  }
  __syncwarp();
  return true;
}

// C (m x m, smem) = alpha * op(X) op(Y) + beta * C, all operands m x m blocks in smem (ld BLD).
// tx: 0 -> X[i][k], 1 -> X[k][i];  ty: 0 -> Y[k][n], 1 -> Y[n][k].
// m = 64: each thread owns rows {2r, 2r+1} and columns {c, c+16, c+32, c+48} (register tile).
template <int M>
__device__ void block_gemm(float* C, const float* X, int tx, const float* Y, int ty, float alpha,
                           float beta) {
  if constexpr (M == 64) {
    const int rb = threadIdx.x >> 4, cb = threadIdx.x & 15;
    float acc[2][4] = {};
#pragma unroll 4
    for (int k = 0; k < M; ++k) {
      float x[2], y[4];
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        const int i = 2 * rb + a;
        x[a] = tx ? X[k * BLD + i] : X[i * BLD + k];
      }
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int n = cb + 16 * b;
        y[b] = ty ? Y[n * BLD + k] : Y[k * BLD + n];
      }
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(x[a], y[b], acc[a][b]);
    }
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        float* cp = C + (2 * rb + a) * BLD + cb + 16 * b;
        *cp = (beta == 0.f) ? alpha * acc[a][b] : fmaf(beta, *cp, alpha * acc[a][b]);
      }
  } else {
    for (int e = threadIdx.x; e < M * M; e += BASE_THREADS) {
      const int i = e / M, n = e % M;
      float acc = 0.f;
#pragma unroll 8
      for (int k = 0; k < M; ++k) {
        const float x = tx ? X[k * BLD + i] : X[i * BLD + k];
        const float y = ty ? Y[n * BLD + k] : Y[k * BLD + n];
        acc = fmaf(x, y, acc);
      }
      C[i * BLD + n] = (beta == 0.f) ? alpha * acc : fmaf(beta, C[i * BLD + n], alpha * acc);
    }
  }
}

constexpr int kLeaf = 16;

template <int N>
__device__ bool base_rec(float* A, float* U, float* V, int o, int32_t* status, int index0,
                         int* fail) {
  if constexpr (N == kLeaf) {
    if (threadIdx.x < 32) {
      if (!leaf<kLeaf>(A, U, V, o, threadIdx.x, status, index0) && threadIdx.x == 0) *fail = 1;
    }
    __syncthreads();
    return *fail == 0;
  } else {
    constexpr int m = N / 2;
    float* Bb = A + o * BLD + o + m;          // A[o:o+m, o+m:o+N]
    float* Aa = A + o * BLD + o;              // A[o:o+m, o:o+m]
    float* U11 = U + o * BLD + o;
    float* U12 = U + o * BLD + o + m;
    float* U22 = U + (o + m) * BLD + o + m;
    if (!base_rec<m>(A, U, V, o + m, status, index0, fail)) return false;
    block_gemm<m>(U12, Bb, 0, U22, 1, 1.f, 0.f);     // T = B U22^T
    __syncthreads();
    block_gemm<m>(Aa, U12, 0, U12, 1, -1.f, 1.f);    // S = A - T T^T
    __syncthreads();
    if (!base_rec<m>(A, U, V, o, status, index0, fail)) return false;
    block_gemm<m>(Bb, U12, 0, U22, 0, 1.f, 0.f);     // V = T U22
    __syncthreads();
    block_gemm<m>(U12, U11, 0, Bb, 0, -1.f, 0.f);    // U12 = -U11 V
    __syncthreads();
    return true;
  }
}

__global__ void __launch_bounds__(BASE_THREADS, 1)
base_block_kernel(const float* __restrict__ Hblk, float* __restrict__ Ublk, int n, int ld,
                  int index0, int32_t* status) {
  extern __shared__ float sm[];
  float* A = sm;
  float* U = sm + BN_ * BLD;
  float* V = sm + 2 * BN_ * BLD;  // 32 x 33 leaf factor
  __shared__ int bad, fail;
  if (threadIdx.x == 0) {
    bad = gptq::status_bad(status) ? 1 : 0;
    fail = 0;
  }
  for (int e = threadIdx.x; e < BN_ * BN_; e += BASE_THREADS) {
    const int i = e / BN_, k = e % BN_;
    float v = 0.f;
    if (i < n && k < n) v = (i <= k) ? Hblk[(long long)i * ld + k] : 0.f;
    else if (i == k) v = 1.f;  // identity padding at the end
    A[i * BLD + k] = v;
    U[i * BLD + k] = 0.f;
  }
  __syncthreads();
  if (bad) return;
  if (!base_rec<BN_>(A, U, V, 0, status, index0, &fail)) return;
  for (int e = threadIdx.x; e < n * n; e += BASE_THREADS) {
    const int i = e / n, k = e % n;
    Ublk[(long long)i * ld + k] = (i <= k) ? U[i * BLD + k] : 0.f;
  }
}

inline int grid_for(long long total) {
  long long g = (total + 255) / 256;
  const long long cap = (long long)gptq_host::num_sms() * 8;
  return (int)(g < 1 ? 1 : (g > cap ? cap : g));
}

}  // namespace

namespace gptq_host {

int prep_permute_sym(const float* H, float* Hp, const int32_t* perm, int d, cudaStream_t stream) {
  permute_sym_kernel<<<grid_for((long long)d * d), 256, 0, stream>>>(H, Hp, perm, d);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int prep_copy_upper(const float* src, float* dst, int d, cudaStream_t stream) {
  copy_upper_kernel<<<grid_for((long long)d * d), 256, 0, stream>>>(src, dst, d);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int prep_act_order(const float* H, int32_t* perm, int d, cudaStream_t stream) {
  act_order_rank_kernel<<<(d + 255) / 256, 256, 0, stream>>>(H, perm, d);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int prep_identity_perm(int32_t* perm, int d, cudaStream_t stream) {
  identity_perm_kernel<<<grid_for(d), 256, 0, stream>>>(perm, d);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int prep_dead_damp(float* H, uint8_t* dead, int d, float percdamp, int32_t* status,
                   cudaStream_t stream) {
  dead_damp_kernel<<<1, 1024, 0, stream>>>(H, dead, d, percdamp, status);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int prep_zero_lower(float* U, int d, cudaStream_t stream) {
  zero_lower_kernel<<<grid_for((long long)d * d), 256, 0, stream>>>(U, d);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

int prep_base_block(float* Hblk, float* Ublk, int n, int ld, int index0, int32_t* status,
                    cudaStream_t stream) {
  const size_t smem = (2 * (size_t)kPrepBase * BLD + 32 * VLD) * sizeof(float);
  if (ensure_smem_attr(reinterpret_cast<const void*>(base_block_kernel), (int)smem) != 0)
    return GPTQ_ERR_CUDA;
  base_block_kernel<<<1, BASE_THREADS, smem, stream>>>(Hblk, Ublk, n, ld, index0, status);
  return cudaGetLastError() == cudaSuccess ? 0 : GPTQ_ERR_CUDA;
}

}  // namespace gptq_host
